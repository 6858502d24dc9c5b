// Factor projection on tcgen05 tensor cores (bf16 in, fp32 accumulate, bf16 out).
//
// Y[T][N] = x[T][D] W_cat[N][D]^T: the six bias-free projections W_A_q/k/v, W_B_q/k/v of
// the TPA module ("【拜读】Tensor Product Attention Is All You Need…" (coreui.cn), 代码
// 类定义与初始化 and 前向传播) as one GEMM.  The epilogue cuts Y into the six factors with
// the page's views and rotates the B_Q and B_K pairs by RoPE at each token's position
// before they are stored (B_K is cached pre-rotated, same page, 关键问题及回答 问题2).
//
// Persistent, warp-specialised, one CTA per SM:
//   warps 0, 10 TMA producers: 128x64 tiles of x (warp 0) and BNx64 tiles of W_cat
//               (warp 10), 128-byte swizzle, into a ring of shared-memory stages.  The
//               copies one thread issues complete one after another (~0.4K cycles each
//               from L2), so each operand has its own issuing thread.
//   warp 1      TMEM allocator and MMA issuer: tcgen05.mma M=128, N=BN, K=16, fp32
//               accumulators double-buffered in TMEM (2 x 256 columns)
//   warps 2..9  epilogue: tcgen05.ld a row per thread (two warps per row quarter,
//               alternate 32-column chunks), RoPE, bf16, 16-byte stores; runs while
//               the MMA warp fills the other accumulator.
// Tensor-bound: 2*T*N*D flops; x and W_cat are read once from HBM (W_cat stays in L2).
#include <algorithm>

#include "tpa_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace tpa {

namespace {
using namespace sm100;

constexpr int BM = 128, BK = 64, kThreads = 352;
constexpr uint32_t kStageA = BM * BK * 2;   // 16 KiB

struct ProjTcArgs {
    int T, N, D, seqlen, Dh, BN, n_tiles_n, n_tiles, k_blocks, stages;
    const float2* cs;
    ProjLayout L;
    int* err;
    uint32_t wait_limit;
};

__device__ __forceinline__ int seg_of(const ProjLayout& L, int c) {
    int s = 0;
#pragma unroll
    for (int i = 1; i < 6; ++i) s += (c >= L.off[i]);
    return s;
}

// Store output columns [c0, min(c0+16, N)) of token t (v already rotated); tkv is the
// token's cache row (cache mode).
__device__ __forceinline__ void store16(const ProjLayout& L, int N, long long t, long long tkv, int c0,
                                        const float (&v)[16], int* err) {
    const int s0 = seg_of(L, c0);
    const int last = min(c0 + 15, N - 1);
    if (c0 + 15 < N && seg_of(L, last) == s0) {
        const int width = L.off[s0 + 1] - L.off[s0];
        const long long row = seg_row(L, s0, t, tkv);
        if (!in_bounds(row >= 0 && row < L.rows[s0], err)) return;
        const long long e = row * width + (c0 - L.off[s0]);
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(L.dst[s0]) + e;
        if ((e & 7) == 0) {
            uint4 w0, w1;
            w0.x = pack_bf16(v[0], v[1]); w0.y = pack_bf16(v[2], v[3]);
            w0.z = pack_bf16(v[4], v[5]); w0.w = pack_bf16(v[6], v[7]);
            w1.x = pack_bf16(v[8], v[9]); w1.y = pack_bf16(v[10], v[11]);
            w1.z = pack_bf16(v[12], v[13]); w1.w = pack_bf16(v[14], v[15]);
            reinterpret_cast<uint4*>(dst)[0] = w0;
            reinterpret_cast<uint4*>(dst)[1] = w1;
            return;
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int c = c0 + j;
        if (c < N) {
            const int s = seg_of(L, c);
            const int width = L.off[s + 1] - L.off[s];
            const long long row = seg_row(L, s, t, tkv);
            if (in_bounds(row >= 0 && row < L.rows[s], err))
                reinterpret_cast<__nv_bfloat16*>(L.dst[s])[row * width + (c - L.off[s])] = __float2bfloat16_rn(v[j]);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
project_tc_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                  const ProjTcArgs a, const SeqParams start) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t stage_b = (uint32_t)a.BN * BK * 2;
    uint8_t* sa = smem;
    uint8_t* sb = sa + (size_t)a.stages * kStageA;
    uint64_t* full = reinterpret_cast<uint64_t*>(sb + (size_t)a.stages * stage_b);
    uint64_t* empty = full + a.stages;
    uint64_t* tfull = empty + a.stages;     // [2] accumulator ready
    uint64_t* tempty = tfull + 2;           // [2] accumulator drained
    uint64_t* fin = tempty + 2;             // MMAs in flight at exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) { mbar_init(&full[s], 2); mbar_init(&empty[s], 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 8); }
        mbar_init(fin, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) { prefetch_tensormap(&tmx); prefetch_tensormap(&tmw); }
    if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lim = a.wait_limit;

    if (warp == 0 || warp == 10) {
        if (lane == 0) {
            // warp 0 stages the x tiles, warp 10 the W_cat tiles; each arrives once per
            // stage with its own byte count
            const bool xs = warp == 0;
            long long it = 0;
            for (int tile = blockIdx.x; tile < a.n_tiles && !*abort; tile += gridDim.x) {
                const int m = tile / a.n_tiles_n, n = tile - m * a.n_tiles_n;
                for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
                    const int s = (int)(it % a.stages);
                    if (it >= a.stages &&
                        !mbar_wait(&empty[s], (uint32_t)((it / a.stages - 1) & 1), lim, a.err, abort))
                        break;
                    if (xs) {
                        mbar_arrive_expect_tx(&full[s], kStageA);
                        tma_load_2d(sa + (size_t)s * kStageA, &tmx, &full[s], kb * BK, m * BM);
                    } else {
                        mbar_arrive_expect_tx(&full[s], stage_b);
                        tma_load_2d(sb + (size_t)s * stage_b, &tmw, &full[s], kb * BK, n * a.BN);
                    }
                }
            }
            // drain: every issued copy lands before the CTA can exit
            for (int s = 0; s < a.stages; ++s) {
                const long long fills = it > s ? (it - s - 1) / a.stages + 1 : 0;
                if (fills > 0) {
                    drain_wait(&full[s], (uint32_t)((fills - 1) & 1));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, a.BN, 0, 0);
            long long it = 0;
            int local = 0;
            for (int tile = blockIdx.x; tile < a.n_tiles && !*abort; tile += gridDim.x, ++local) {
                const int buf = local & 1;
                if (local >= 2 &&
                    !mbar_wait(&tempty[buf], (uint32_t)(((local >> 1) - 1) & 1), lim, a.err, abort))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)buf * 256u;
                bool ok = true;
                for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
                    const int s = (int)(it % a.stages);
                    if (!mbar_wait(&full[s], (uint32_t)((it / a.stages) & 1), lim, a.err, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sa + (size_t)s * kStageA);
                    const uint32_t b_base = smem_u32(sb + (size_t)s * stage_b);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        mma_ss(d_tmem, smem_desc(a_base + k * 32, 16, 1024, kSwizzle128),
                               smem_desc(b_base + k * 32, 16, 1024, kSwizzle128), idesc,
                               (kb | k) != 0);
                    }
                    mma_commit(&empty[s]);
                }
                if (!ok) break;
                mma_commit(&tfull[buf]);
            }
            // every MMA issued has completed before TMEM is released
            mma_commit(fin);
            drain_wait(fin, 0);
        }
    } else {
        // 8 epilogue warps: warp w reads TMEM lanes 32*(w%4).. (its rows) and every
        // other 32-column chunk of the tile, starting at chunk (w-2)/4.
        const int quarter = warp & 3;
        const int colhalf = (warp - 2) >> 2;
        const int row = quarter * 32 + lane;
        const int half = a.Dh >> 1;
        int local = 0;
        for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++local) {
            const int buf = local & 1;
            // leave together: tcgen05.ld below needs every lane
            const bool got = mbar_wait(&tfull[buf], (uint32_t)((local >> 1) & 1), lim, a.err, abort);
            if (__any_sync(0xffffffffu, !got)) break;
            tc_fence_after();
            const int m = tile / a.n_tiles_n, n = tile - m * a.n_tiles_n;
            const long long t = (long long)m * BM + row;
            const bool valid = t < a.T;
            int pos = 0;
            long long tkv = 0;
            if (valid) {
                const int b = (int)(t / a.seqlen);
                const int i = (int)(t - (long long)b * a.seqlen);
                pos = start.v[b] + i;
                tkv = (long long)b * a.L.kv_cap + pos;
                // cache mode: the sequence's last token records the new length, once
                if (a.L.lengths && n == 0 && colhalf == 0 && i == a.seqlen - 1 &&
                    in_bounds(b < a.L.n_lengths, a.err))
                    a.L.lengths[b] = pos + 1;
            }
            const int col0 = n * a.BN;
            const int cend = min(a.N, col0 + a.BN);
            for (int c = 32 * colhalf; col0 + c < cend; c += 64) {
                const int cg = col0 + c;
                // RoPE cos/sin for the pairs of this chunk, fetched before the TMEM read
                float2 rot[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int cc = cg + 2 * j;
                    const int sg = seg_of(a.L, cc);
                    rot[j] = make_float2(1.f, 0.f);
                    if (valid && (sg == 3 || sg == 4) && cc < cend && in_bounds(pos < a.L.cs_rows, a.err)) {
                        const int kp = ((cc - a.L.off[sg]) % a.Dh) >> 1;
                        rot[j] = __ldg(&a.cs[(long long)pos * half + kp]);
                    }
                }
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)buf * 256u + c, r);
                tmem_ld_wait();
                if (!valid) continue;
                float v[32];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float x0 = __uint_as_float(r[2 * j]), x1 = __uint_as_float(r[2 * j + 1]);
                    v[2 * j] = x0 * rot[j].x - x1 * rot[j].y;
                    v[2 * j + 1] = x0 * rot[j].y + x1 * rot[j].x;
                }
                store16(a.L, cend, t, tkv, cg, *reinterpret_cast<float(*)[16]>(&v[0]), a.err);
                if (cg + 16 < cend) store16(a.L, cend, t, tkv, cg + 16, *reinterpret_cast<float(*)[16]>(&v[16]), a.err);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

int pick_bn(int N, int T) {
    int best_bn = 256, best_waste = 1 << 30;
    const int nt0 = (N + 255) / 256;
    for (int nt = nt0; nt <= nt0 + 3; ++nt) {
        int bn = (N + nt - 1) / nt;
        bn = (bn + 15) / 16 * 16;
        if (bn > 256 || bn < 16) continue;
        const int waste = nt * bn - N;
        if (waste < best_waste) { best_waste = waste; best_bn = bn; }
    }
    // Few row tiles (small batches, e.g. one decode token per sequence): narrower column
    // tiles spread the weight stream over more SMs instead of a handful of CTAs.
    const long long m_tiles = (T + BM - 1) / BM, sms = sm_count();
    if (m_tiles * ((N + best_bn - 1) / best_bn) < sms) {
        int bn = (int)((N * m_tiles + sms - 1) / sms);
        bn = std::max(16, (bn + 15) / 16 * 16);
        best_bn = std::min(best_bn, bn);
    }
    return best_bn;
}
}  // namespace

bool project_tc_supported(const Shape& s, int T) {
    return s.bf16 && s.D % 8 == 0 && s.D >= 8 && T >= 1;
}

cudaError_t launch_project_tc(const Shape& s, const void* x, const void* w, int batch, int seqlen,
                              const SeqParams& start, const float* cs, const ProjLayout& L,
                              int* err, uint32_t wait_limit, cudaStream_t st) {
    ProjTcArgs a;
    a.T = batch * seqlen;
    a.N = L.off[6];
    a.D = s.D;
    a.seqlen = seqlen;
    a.Dh = s.Dh;
    a.BN = pick_bn(a.N, a.T);
    a.n_tiles_n = (a.N + a.BN - 1) / a.BN;
    a.n_tiles = ((a.T + BM - 1) / BM) * a.n_tiles_n;
    a.k_blocks = (a.D + BK - 1) / BK;
    const uint32_t stage_bytes = kStageA + (uint32_t)a.BN * BK * 2;
    a.stages = std::min(6, (int)((220u * 1024u) / stage_bytes));
    a.cs = reinterpret_cast<const float2*>(cs);
    a.L = L;
    a.err = err;
    a.wait_limit = wait_limit;

    CUtensorMap tmx, tmw;
    const uint64_t dx[2] = {(uint64_t)a.D, (uint64_t)a.T};
    const uint64_t dw[2] = {(uint64_t)a.D, (uint64_t)a.N};
    const uint64_t stride[1] = {(uint64_t)a.D * 2};
    const uint32_t bx[2] = {BK, BM};
    const uint32_t bw[2] = {BK, (uint32_t)a.BN};
    if (!make_tmap_bf16(&tmx, x, 2, dx, stride, bx) || !make_tmap_bf16(&tmw, w, 2, dw, stride, bw))
        return cudaErrorInvalidValue;

    const size_t smem = 1024 + (size_t)a.stages * stage_bytes + (2 * a.stages + 5) * 8 + 16;
    cudaError_t e = allow_smem(reinterpret_cast<const void*>(project_tc_kernel), (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = std::min(a.n_tiles, sm_count());
    project_tc_kernel<<<grid, kThreads, smem, st>>>(tmx, tmw, a, start);
    return cudaGetLastError();
}

}  // namespace tpa
