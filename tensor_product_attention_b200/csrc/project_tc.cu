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
//               alternate 32-column chunks), RoPE, bf16, into a 32 x 32 tile in shared
//               memory that one lane writes out with a TMA tensor store (double-buffered
//               per warp); a chunk that straddles two factors or two sequences, or a
//               factor whose rows are not 16-byte aligned, goes out through coalesced
//               stores instead (four lanes per 64-byte row piece).  The RoPE cos/sin of
//               a chunk are 16-byte loads, kept while the next chunk needs the same
//               pairs.  Runs while the MMA warp fills the other accumulator.
// The single-thread loops keep their ring position as 32-bit stage/phase counters: a
// 64-bit modulo per k-block cost the MMA issuer more than half of the tensor rate.
// Counted against the tensor peak (2*T*N*D flops); x and W_cat are read once from HBM
// (W_cat stays in L2).  At 128x160 tiles the main loop runs near the shared-memory port
// bound instead: per k-block the SM takes 36 KB of TMA writes and serves 36 KB of MMA
// operand reads, ~576 cycles at 128 B/clk against 320 of MMA.
#include <algorithm>
#include <cstring>

#include "tpa_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace tpa {

namespace {
using namespace sm100;

constexpr int BM = 128, BK = 64, kThreads = 352;
constexpr uint32_t kStageA = BM * BK * 2;   // 16 KiB
constexpr uint32_t kOutStage = 32 * 64;     // one 32 rows x 32 bf16 output tile
constexpr int kEpiWarps = 8;                // each with two output tiles

// Output tensor maps of the six factors ([rows][width] bf16, box 32 x 32, no swizzle);
// bit s of `mask` says that factor s may be written by TMA.
struct OutMaps {
    CUtensorMap m[6];
    uint32_t mask;
};

struct ProjTcArgs {
    int T, N, D, seqlen, Dh, BN, n_tiles_n, n_tiles, k_blocks, stages;
    int cs_vec;     // RoPE table 16-byte aligned with an even number of pairs per row
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

// Store output columns [c0, min(c0+8, cend)) of token t from 8 packed bf16.
__device__ __forceinline__ void store8(const ProjLayout& L, int cend, long long t, long long tkv, int c0,
                                       uint4 w, int* err) {
    const int s0 = seg_of(L, c0);
    if (c0 + 7 < cend && seg_of(L, c0 + 7) == s0) {
        const int width = L.off[s0 + 1] - L.off[s0];
        const long long row = seg_row(L, s0, t, tkv);
        if (!in_bounds(row >= 0 && row < L.rows[s0], err)) return;
        const long long e = row * width + (c0 - L.off[s0]);
        if ((e & 7) == 0) {
            *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(L.dst[s0]) + e) = w;
            return;
        }
    }
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int c = c0 + j;
        if (c < cend) {
            const int s = seg_of(L, c);
            const int width = L.off[s + 1] - L.off[s];
            const long long row = seg_row(L, s, t, tkv);
            if (in_bounds(row >= 0 && row < L.rows[s], err)) {
                const uint16_t bits = (uint16_t)((j & 1) ? (wv[j >> 1] >> 16) : (wv[j >> 1] & 0xffffu));
                reinterpret_cast<uint16_t*>(L.dst[s])[row * width + (c - L.off[s])] = bits;
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
project_tc_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                  const __grid_constant__ OutMaps om, const ProjTcArgs a, const SeqParams start) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t stage_b = (uint32_t)a.BN * BK * 2;
    uint8_t* sa = smem;
    uint8_t* sb = sa + (size_t)a.stages * kStageA;
    uint8_t* ostage = sb + (size_t)a.stages * stage_b;   // kEpiWarps x 2 x kOutStage
    uint64_t* full = reinterpret_cast<uint64_t*>(ostage + kEpiWarps * 2 * kOutStage);
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
            int it = 0, s = 0;        // copies issued; ring slot it % stages
            uint32_t ph = 0;          // (it / stages) & 1
            for (int tile = blockIdx.x; tile < a.n_tiles && !*abort; tile += gridDim.x) {
                const int m = tile / a.n_tiles_n, n = tile - m * a.n_tiles_n;
                bool ok = true;
                for (int kb = 0; kb < a.k_blocks; ++kb) {
                    if (it >= a.stages && !mbar_wait(&empty[s], ph ^ 1u, lim, a.err, abort)) {
                        ok = false;
                        break;
                    }
                    if (xs) {
                        mbar_arrive_expect_tx(&full[s], kStageA);
                        tma_load_2d(sa + (size_t)s * kStageA, &tmx, &full[s], kb * BK, m * BM);
                    } else {
                        mbar_arrive_expect_tx(&full[s], stage_b);
                        tma_load_2d(sb + (size_t)s * stage_b, &tmw, &full[s], kb * BK, n * a.BN);
                    }
                    ++it;
                    if (++s == a.stages) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
            }
            // drain: every issued copy lands before the CTA can exit
            for (int s = 0; s < a.stages; ++s) {
                const int fills = it > s ? (it - s - 1) / a.stages + 1 : 0;
                if (fills > 0) {
                    drain_wait(&full[s], (uint32_t)((fills - 1) & 1));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(BM, a.BN, 0, 0);
            int s = 0;                // ring slot
            uint32_t ph = 0;          // phase parity of the slot's current fill
            int local = 0;
            for (int tile = blockIdx.x; tile < a.n_tiles && !*abort; tile += gridDim.x, ++local) {
                const int buf = local & 1;
                if (local >= 2 &&
                    !mbar_wait(&tempty[buf], (uint32_t)(((local >> 1) - 1) & 1), lim, a.err, abort))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)buf * 256u;
                bool ok = true;
                for (int kb = 0; kb < a.k_blocks; ++kb) {
                    if (!mbar_wait(&full[s], ph, lim, a.err, abort)) {
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
                    if (++s == a.stages) { s = 0; ph ^= 1u; }
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
        const bool cache_mode = a.L.kv_cap > 0;
        // this warp's two output tiles (row-major, 64 bytes a row); a TMA store reads the
        // one it was given while the warp fills the other
        uint8_t* const obuf = ostage + (size_t)(warp - 2) * 2 * kOutStage;
        int nb = 0;   // TMA stores issued by this warp (lane 0)
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
            // the warp's 32 rows: tokens t0..t0+31; cache rows are consecutive only when all
            // 32 tokens exist and belong to one sequence
            const long long t0 = (long long)m * BM + quarter * 32;
            const bool kv_rows_ok = t0 + 31 < a.T && t0 / a.seqlen == (t0 + 31) / a.seqlen;
            const long long tkv0 = __shfl_sync(0xffffffffu, tkv, 0);
            const int col0 = n * a.BN;
            const int cend = min(a.N, col0 + a.BN);
            int rot_key = -1;     // first RoPE pair held in rot[], -1 if none
            float2 rot[16];
            for (int c = 32 * colhalf; col0 + c < cend && t0 < a.T; c += 64) {
                const int cg = col0 + c;
                const int s0 = seg_of(a.L, cg);
                const bool whole = cg + 31 < cend && seg_of(a.L, cg + 31) == s0;
                const int o = cg - a.L.off[s0];
                const bool rseg = s0 == 3 || s0 == 4;
                bool do_rot = true;
                if (whole && !rseg) {
                    do_rot = false;
                } else if (whole && a.cs_vec && (o % a.Dh) + 32 <= a.Dh && ((o % a.Dh) & 3) == 0) {
                    // 16 consecutive pairs from the token's table row
                    const int kp0 = (o % a.Dh) >> 1;
                    if (kp0 != rot_key) {
                        rot_key = kp0;
                        if (valid && in_bounds(pos < a.L.cs_rows, a.err)) {
                            const float4* src = reinterpret_cast<const float4*>(a.cs + (long long)pos * half + kp0);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float4 v = __ldg(src + q);
                                rot[2 * q] = make_float2(v.x, v.y);
                                rot[2 * q + 1] = make_float2(v.z, v.w);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j) rot[j] = make_float2(1.f, 0.f);
                        }
                    }
                } else {
                    rot_key = -1;
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
                }
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)buf * 256u + c, r);
                tmem_ld_wait();
                const bool kv_seg = cache_mode && s0 != 0 && s0 != 3;
                const bool tma = whole && ((om.mask >> s0) & 1u) && (o & 7) == 0 && (!kv_seg || kv_rows_ok);
                // the tile written two TMA stores ago has been read by then
                uint8_t* const cur = obuf + (size_t)(nb & 1) * kOutStage;
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
                const uint32_t cu32 = smem_u32(cur);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float v[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float x0 = __uint_as_float(r[8 * u + 2 * j]), x1 = __uint_as_float(r[8 * u + 2 * j + 1]);
                        if (do_rot) {
                            const float2 cr = rot[4 * u + j];
                            v[2 * j] = x0 * cr.x - x1 * cr.y;
                            v[2 * j + 1] = x0 * cr.y + x1 * cr.x;
                        } else {
                            v[2 * j] = x0;
                            v[2 * j + 1] = x1;
                        }
                    }
                    uint4 w;
                    w.x = pack_bf16(v[0], v[1]); w.y = pack_bf16(v[2], v[3]);
                    w.z = pack_bf16(v[4], v[5]); w.w = pack_bf16(v[6], v[7]);
                    sts_v4(cu32 + (uint32_t)lane * 64u + (uint32_t)u * 16u, w);
                }
                if (tma) {
                    // rows past T fall outside the factor's tensor map and are not written
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&om.m[s0], cur, o, (int)(kv_seg ? tkv0 : t0));
                        bulk_commit_group();
                    }
                    ++nb;
                } else {
                    __syncwarp();
                    asm volatile("" ::: "memory");
                    // lanes 4i..4i+3 cover one row's 64 bytes, 8 rows per pass
#pragma unroll
                    for (int pass = 0; pass < 4; ++pass) {
                        const int rr = 8 * pass + (lane >> 2), u = lane & 3;
                        const long long tr = t0 + rr;
                        const long long tkv_r = __shfl_sync(0xffffffffu, tkv, rr);
                        const int cu = cg + 8 * u;
                        if (tr < a.T && cu < cend) {
                            const uint4 w = lds_v4(cu32 + (uint32_t)rr * 64u + (uint32_t)u * 16u);
                            store8(a.L, cend, tr, tkv_r, cu, w, a.err);
                        }
                    }
                    __syncwarp();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
        }
        // every TMA store has written its tile before the CTA exits
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
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
    // 227 KB per CTA: 1 KB for alignment, the barriers, the epilogue's output tiles
    const uint32_t budget = 232448u - 1024u - 256u - kEpiWarps * 2u * kOutStage;
    a.stages = std::min(6, (int)(budget / stage_bytes));
    a.cs = reinterpret_cast<const float2*>(cs);
    a.cs_vec = (reinterpret_cast<uintptr_t>(cs) % 16 == 0 && (s.Dh / 2) % 2 == 0) ? 1 : 0;
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

    // output maps: factors with 16-byte aligned rows and base, at least one 32-column box wide
    OutMaps om;
    om.mask = 0;
    for (int f = 0; f < 6; ++f) {
        const int width = L.off[f + 1] - L.off[f];
        std::memset(&om.m[f], 0, sizeof(CUtensorMap));
        if (width < 32 || width % 8 != 0 || L.rows[f] < 1 || !L.dst[f] ||
            reinterpret_cast<uintptr_t>(L.dst[f]) % 16 != 0)
            continue;
        const uint64_t dd[2] = {(uint64_t)width, (uint64_t)L.rows[f]};
        const uint64_t ds[1] = {(uint64_t)width * 2};
        const uint32_t bo[2] = {32, 32};
        if (make_tmap_bf16(&om.m[f], L.dst[f], 2, dd, ds, bo, 0)) om.mask |= 1u << f;
    }
    const size_t smem = 1024 + (size_t)a.stages * stage_bytes + kEpiWarps * 2 * kOutStage + (2 * a.stages + 5) * 8 + 16;
    cudaError_t e = allow_smem(reinterpret_cast<const void*>(project_tc_kernel), (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = std::min(a.n_tiles, sm_count());
    project_tc_kernel<<<grid, kThreads, smem, st>>>(tmx, tmw, om, a, start);
    return cudaGetLastError();
}

}  // namespace tpa
