// Causal prefill from the factor cache on tcgen05 tensor cores (bf16, fp32 accumulate).
//
// The TPA attention of "【拜读】Tensor Product Attention Is All You Need…" (coreui.cn),
// §3 公式描述 and 代码 前向传播, evaluated from the cached factors (B_K already rotated,
// same page, 关键问题及回答 问题2); attention softmax(QK^T/sqrt(d_h))V per the jieyibu.net
// TPA page, Ⅱ.1.  K and V are never formed in device memory.
//
// Rows of the MMAs are (query, head) pairs, so every tensor-core operand that comes from
// the cache is shared by all heads:
//   q~_{i,h}  = log2(e)/(R_Q R_K sqrt(d_h)) * sum_r a^Q_{i,h,r} b^Q_{i,r}     (prologue)
//   U         = q~ . b^K_{j,s}^T              tcgen05, M=128 rows (i,h), N=KT*R (j,s), K=d_h
//   score     = sum_s a^K_{j,h,s} U_{(i,h),(j,s)}                 CUDA cores, per row
//   W         = exp2(score - m) * a^V_{j,h,s}  (online softmax, bf16, written to TMEM)
//   O        += W . b^V                       tcgen05, A=W from TMEM, B=b^V (MN-major)
//   out_{i,h} = O / (l * R_V)
// The a^Q half of the per-head weighting is applied once per query (folding it into
// q~) instead of once per (query, key) pair: the same sums, reassociated.
//
// One CTA = 256 rows (two 128-row M-blocks: 256/h queries x h heads) of one sequence,
// walking key tiles of KT = 128/R keys.  Warp roles:
//   warp 0     TMA: b^K, b^V tiles (2-D maps over the cache, 128-byte swizzle) and
//              a^K, a^V tiles (bulk copies) into a ring of stages
//   warp 1     TMEM owner (512 columns) and MMA issuer; the two M-blocks ping-pong so
//              that one block's softmax overlaps the other block's MMAs
//   warps 4-11 softmax for M-block 0 (warps 4-7) and 1 (warps 8-11), one row per thread
// The control warpgroup (warps 0-3) hands registers to the softmax warpgroups with
// setmaxnreg once the prologue is done.
// TMEM: U_0 [0,128), U_1 [128,256), O_0 and O_1 after 256 (d_h columns each); W_b
// overwrites the first half of U_b once the scores are read (bf16 pairs).
#include <algorithm>
#include <cmath>

#include "tpa_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace tpa {

namespace {
using namespace sm100;

constexpr int kThreads = 384;   // 3 warpgroups: TMA/MMA, softmax block 0, softmax block 1
constexpr int kRegsCtl = 96, kRegsSoftmax = 200;   // 128*96 + 256*200 = 63488 <= 384*168 (launch)
constexpr uint32_t kBox = 128 * 128;        // one TMA box: 128 rows x 128 bytes
constexpr float kRescale = 8.f;             // lazy rescale threshold (log2 units)

struct PrefillTcArgs {
    const __nv_bfloat16* a_q;     // [T][H][Rq]
    const __nv_bfloat16* b_q;     // [T][Rq][DH]
    const __nv_bfloat16* ca_k;    // [B][cap][H][R]
    const __nv_bfloat16* ca_v;
    __nv_bfloat16* out;           // [T][H][DH]
    int S, H, Rq, cap, n_qblocks, qpb, stages;
    uint32_t a_bytes;             // bytes of one a^K (or a^V) tile: KT*H*R*2
    uint32_t stage_bytes;
    float qscale, out_scale;
    int* err;
    uint32_t wait_limit;
};

// R consecutive bf16 factor values at element offset idx*R (R = 1, 2 or 4).
template <int R>
__device__ __forceinline__ void load_r(const __nv_bfloat16* base, int idx, float (&f)[R]) {
    if constexpr (R == 1) {
        f[0] = __bfloat162float(base[idx]);
    } else if constexpr (R == 2) {
        const uint32_t w = reinterpret_cast<const uint32_t*>(base)[idx];
        f[0] = bf16lo(w); f[1] = bf16hi(w);
    } else {
        const uint2 w = reinterpret_cast<const uint2*>(base)[idx];
        f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
    }
}

// One pass of the softmax over a key tile for this thread's row (i, h), relative to a
// reference max m_ref: d_j = sum_s a^K_{j,h,s} U_{(j,s)} - m_ref (log2 units), mx =
// max_j d_j, p_j = 2^d_j, lsum = sum_j p_j, and the W row (p_j a^V_{j,h,s}) in K order
// (j, s) packed as bf16 pairs.  MASKED applies the causal bound j <= p_i (diagonal tiles).
template <int R, bool MASKED, int HS_>
__device__ __forceinline__ void softmax_pass(uint32_t u_addr, const __nv_bfloat16* ak,
                                             const __nv_bfloat16* av, int H, int h, int j0, int p_i,
                                             float m_ref, float& mx, float& lsum, uint32_t (&wp)[64]) {
    const int HS = HS_ > 0 ? HS_ : H;   // head count, compile-time when known
    mx = -INFINITY;
    lsum = 0.f;
    if constexpr (R == 2) {
        // one 32-bit word holds a key's two factor values; W = bf16x2(p) * (a^V pair).
        // Four independent max/sum accumulators keep the loop-carried chains short.
        const uint32_t* akr = reinterpret_cast<const uint32_t*>(ak) + h;
        const uint32_t* avr = reinterpret_cast<const uint32_t*>(av) + h;
        float mxa[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float lsa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            uint32_t u[64];
            tmem_ld32(u_addr + (uint32_t)hf * 64u, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
            tmem_ld32(u_addr + (uint32_t)hf * 64u + 32u, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
            uint32_t wa[32], wv[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                wa[q] = akr[(hf * 32 + q) * HS];
                wv[q] = avr[(hf * 32 + q) * HS];
            }
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int jj = hf * 32 + q;
                float d = fmaf(bf16lo(wa[q]), __uint_as_float(u[2 * q]), -m_ref);
                d = fmaf(bf16hi(wa[q]), __uint_as_float(u[2 * q + 1]), d);
                if (MASKED) d = (j0 + jj <= p_i) ? d : -INFINITY;
                mxa[q & 3] = fmaxf(mxa[q & 3], d);
                const float p = ex2(d);
                lsa[q & 3] += p;
                const __nv_bfloat162 pw = __float2bfloat162_rn(p);
                const __nv_bfloat162 prod = __hmul2(pw, *reinterpret_cast<const __nv_bfloat162*>(&wv[q]));
                uint32_t w = *reinterpret_cast<const uint32_t*>(&prod);
                if (MASKED) w = (p != 0.f) ? w : 0u;
                wp[jj] = w;
            }
        }
        mx = fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3]));
        lsum = (lsa[0] + lsa[1]) + (lsa[2] + lsa[3]);
        return;
    }
    constexpr int KPH = 64 / R;          // keys per 64 U columns
    float wprev = 0.f;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        uint32_t u[64];
        tmem_ld32(u_addr + (uint32_t)hf * 64u, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
        tmem_ld32(u_addr + (uint32_t)hf * 64u + 32u, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < KPH; ++q) {
            const int jj = hf * KPH + q;
            float fa[R], fv[R];
            load_r<R>(ak, jj * HS + h, fa);
            float d = -m_ref;
#pragma unroll
            for (int sr = 0; sr < R; ++sr) d = fmaf(fa[sr], __uint_as_float(u[q * R + sr]), d);
            if (MASKED) d = (j0 + jj <= p_i) ? d : -INFINITY;
            mx = fmaxf(mx, d);
            const float p = ex2(d);
            lsum += p;
            load_r<R>(av, jj * HS + h, fv);
#pragma unroll
            for (int sr = 0; sr < R; ++sr) {
                float w = p * fv[sr];
                if (MASKED) w = (p != 0.f) ? w : 0.f;
                const int k = jj * R + sr;
                if (k & 1) wp[k >> 1] = pack_bf16(wprev, w);
                else wprev = w;
            }
        }
    }
}

template <int DH, int R, int HC>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  const PrefillTcArgs a, const SeqParams start) {
    constexpr int KT = 128 / R;            // keys per tile
    constexpr int NB = DH / 64;            // 64-wide column blocks of d_h
    constexpr uint32_t kQBytes = NB * 256u * 128u;
    constexpr int UW = KT * R;             // U columns per M-block (= 128)

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sq = smem;                                   // q~, [NB][256 rows][128 B]
    uint8_t* stg = smem + kQBytes;                        // stages
    uint64_t* bars = reinterpret_cast<uint64_t*>(stg + (size_t)a.stages * a.stage_bytes);
    uint64_t* kv_full = bars;
    uint64_t* kv_empty = kv_full + a.stages;
    uint64_t* u_ready = kv_empty + a.stages;    // [2]
    uint64_t* w_ready = u_ready + 2;            // [2]
    uint64_t* o_done = w_ready + 2;             // [2]
    uint64_t* fin = o_done + 2;                 // MMAs in flight at exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = HC > 0 ? HC : a.H;
    const int qb = a.n_qblocks - 1 - (int)blockIdx.x;   // longest rows first
    const int b = blockIdx.y;
    const int q0 = qb * a.qpb;
    const int nq = min(a.qpb, a.S - q0);
    const int p0 = start.v[b] + q0;
    const int p_last = p0 + nq - 1;
    const int n_tiles = p_last / KT + 1;
    const int kv_len = start.v[b] + a.S;
    const uint32_t lim = a.wait_limit;

    auto stage_bk = [&](int s) { return stg + (size_t)s * a.stage_bytes; };
    auto stage_bv = [&](int s) { return stg + (size_t)s * a.stage_bytes + NB * kBox; };
    auto stage_ak = [&](int s) {
        return reinterpret_cast<const __nv_bfloat16*>(stg + (size_t)s * a.stage_bytes + 2 * NB * kBox);
    };
    auto stage_av = [&](int s) {
        return reinterpret_cast<const __nv_bfloat16*>(stg + (size_t)s * a.stage_bytes + 2 * NB * kBox +
                                                      ((a.a_bytes + 127u) & ~127u));
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&u_ready[i], 1);
            mbar_init(&w_ready[i], 128);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(fin, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) { prefetch_tensormap(&tmk); prefetch_tensormap(&tmv); }
    if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }

    // ---- prologue: q~ rows (bf16, 128-byte swizzled K-major) by the 256 softmax threads
    if (warp >= 4) {
        const int row = threadIdx.x - 128;                // 0..255
        const int i_loc = row / H, h = row - (row / H) * H;
        const bool vq = i_loc < nq;
        const long long t = (long long)b * a.S + q0 + (vq ? i_loc : 0);
        float aq[16];
        for (int r = 0; r < a.Rq; ++r) aq[r] = vq ? __bfloat162float(a.a_q[(t * H + h) * a.Rq + r]) * a.qscale : 0.f;
        const __nv_bfloat16* bq = a.b_q + t * a.Rq * DH;
#pragma unroll 1
        for (int k8 = 0; k8 < DH; k8 += 8) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (vq) {
                for (int r = 0; r < a.Rq; ++r) {
                    const uint4 raw = *reinterpret_cast<const uint4*>(bq + r * DH + k8);
                    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(p2[e]);
                        acc[2 * e] = fmaf(aq[r], f.x, acc[2 * e]);
                        acc[2 * e + 1] = fmaf(aq[r], f.y, acc[2 * e + 1]);
                    }
                }
            }
            uint4 w;
            w.x = pack_bf16(acc[0], acc[1]); w.y = pack_bf16(acc[2], acc[3]);
            w.z = pack_bf16(acc[4], acc[5]); w.w = pack_bf16(acc[6], acc[7]);
            const int cb = k8 >> 6;
            *reinterpret_cast<uint4*>(sq + cb * (256u * 128u) + sw128_offset(row, (k8 & 63) * 2)) = w;
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp < 4) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
      if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint32_t full_bytes = 2u * NB * kBox;
            int t = 0;
            for (; t < n_tiles && !*abort; ++t) {
                const int s = t % a.stages;
                if (t >= a.stages &&
                    !mbar_wait(&kv_empty[s], (uint32_t)((t / a.stages - 1) & 1), lim, a.err, abort))
                    break;
                const int j0 = t * KT;
                const int rows_a = min(KT, a.cap - j0);
                const uint32_t abytes = (uint32_t)rows_a * H * R * 2u;
                mbar_arrive_expect_tx(&kv_full[s], full_bytes + 2u * abytes);
                const int y = (int)(((long long)b * a.cap + j0) * R);
#pragma unroll
                for (int cb = 0; cb < NB; ++cb) {
                    tma_load_2d(stage_bk(s) + cb * kBox, &tmk, &kv_full[s], cb * 64, y);
                    tma_load_2d(stage_bv(s) + cb * kBox, &tmv, &kv_full[s], cb * 64, y);
                }
                const long long ea = ((long long)b * a.cap + j0) * H * R;
                bulk_load((void*)stage_ak(s), a.ca_k + ea, abytes, &kv_full[s]);
                bulk_load((void*)stage_av(s), a.ca_v + ea, abytes, &kv_full[s]);
            }
            for (int s = 0; s < a.stages; ++s) {          // drain issued copies
                const int fills = t > s ? (t - s - 1) / a.stages + 1 : 0;
                if (fills > 0)
                    drain_wait(&kv_full[s], (uint32_t)((fills - 1) & 1));
            }
        }
      } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_bf16(128, UW, 0, 0);
            const uint32_t idesc_pv = idesc_bf16(128, DH, 0, 1);
            const uint32_t q_base = smem_u32(sq);
            for (int t = 0; t <= n_tiles && !*abort; ++t) {
                const int s = t % a.stages;
                if (t < n_tiles) {
                    if (!mbar_wait(&kv_full[s], (uint32_t)((t / a.stages) & 1), lim, a.err, abort)) break;
                    tc_fence_after();
                }
                bool ok = true;
                for (int bl = 0; bl < 2; ++bl) {
                    const uint32_t u_col = tmem + (uint32_t)bl * 128u;
                    const uint32_t o_col = tmem + 256u + (uint32_t)bl * DH;
                    if (t > 0) {
                        // O_bl += W_bl(t-1) . b^V(t-1)
                        if (!mbar_wait(&w_ready[bl], (uint32_t)((t - 1) & 1), lim, a.err, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const int sp = (t - 1) % a.stages;
                        const uint32_t bv = smem_u32(stage_bv(sp));
#pragma unroll
                        for (int k = 0; k < UW / 16; ++k)
                            mma_ts(o_col, u_col + (uint32_t)k * 8u,
                                   smem_desc(bv + (uint32_t)k * 2048u, kBox, 1024, kSwizzle128),
                                   idesc_pv, (t - 1 > 0 || k > 0) ? 1u : 0u);
                        if (bl == 1) mma_commit(&kv_empty[sp]);
                        if (t == n_tiles) mma_commit(&o_done[bl]);
                    }
                    if (t < n_tiles) {
                        // U_bl = q~_bl . b^K(t)^T
                        const uint32_t bk = smem_u32(stage_bk(s));
#pragma unroll
                        for (int k = 0; k < DH / 16; ++k) {
                            const uint32_t cb = (uint32_t)(k >> 2), kk = (uint32_t)(k & 3) * 32u;
                            mma_ss(u_col,
                                   smem_desc(q_base + cb * 256u * 128u + (uint32_t)bl * 128u * 128u + kk,
                                             16, 1024, kSwizzle128),
                                   smem_desc(bk + cb * kBox + kk, 16, 1024, kSwizzle128), idesc_qk,
                                   k > 0 ? 1u : 0u);
                        }
                        mma_commit(&u_ready[bl]);
                    }
                }
                if (!ok) break;
            }
            // every MMA issued has completed before TMEM is released
            mma_commit(fin);
            drain_wait(fin, 0);
        }
      }
    } else {
        // ------------------------------------------------------------ softmax
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        const int bl = (warp - 4) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;                 // TMEM lane
        const int row = bl * 128 + r;
        const int i_loc = row / H, h = row - (row / H) * H;
        const bool vq = i_loc < nq;
        const int p_i = p0 + min(i_loc, nq - 1);
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t u_col = (uint32_t)bl * 128u;
        const uint32_t o_col = 256u + (uint32_t)bl * DH;
        float m_use = -INFINITY, l = 0.f;
        bool alive = true;
        const uint32_t u_addr = lane_addr + u_col;
        for (int t = 0; t < n_tiles; ++t) {
            // leave together: the warp votes below need every lane
            const bool got = mbar_wait(&u_ready[bl], (uint32_t)(t & 1), lim, a.err, abort);
            if (__any_sync(0xffffffffu, !got)) { alive = false; break; }
            tc_fence_after();
            const int s = t % a.stages;
            const int j0 = t * KT;
            const __nv_bfloat16* ak = stage_ak(s);
            const __nv_bfloat16* av = stage_av(s);
            const bool masked = j0 + KT - 1 > p0;        // same for every row of the CTA
            uint32_t wp[64];
            float mx = -INFINITY, lsum = 0.f;
            bool ok = false;
            if (t > 0) {
                // common case: one pass against the running max
                if (masked) softmax_pass<R, true, HC>(u_addr, ak, av, H, h, j0, p_i, m_use, mx, lsum, wp);
                else softmax_pass<R, false, HC>(u_addr, ak, av, H, h, j0, p_i, m_use, mx, lsum, wp);
                ok = mx <= kRescale;
            }
            if (__all_sync(0xffffffffu, ok)) {
                l += lsum;
            } else {
                // first tile, or the max rose by more than 2^kRescale: exact max, rescale O
                if (t == 0) {
                    if (masked) softmax_pass<R, true, HC>(u_addr, ak, av, H, h, j0, p_i, 0.f, mx, lsum, wp);
                    else softmax_pass<R, false, HC>(u_addr, ak, av, H, h, j0, p_i, 0.f, mx, lsum, wp);
                }
                const float m_new = (t == 0) ? mx : (mx > kRescale ? m_use + mx : m_use);
                const float alpha = (t == 0) ? 1.f : ex2(m_use - m_new);
                if (t > 0) l *= alpha;
                if (t > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                    // O row *= alpha (PV(t-1) has completed: QK(t) was committed after it)
#pragma unroll
                    for (int c = 0; c < DH / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(lane_addr + o_col + (uint32_t)c * 32u, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(lane_addr + o_col + (uint32_t)c * 32u, o);
                    }
                    tmem_st_wait();
                }
                m_use = m_new;
                if (masked) softmax_pass<R, true, HC>(u_addr, ak, av, H, h, j0, p_i, m_use, mx, lsum, wp);
                else softmax_pass<R, false, HC>(u_addr, ak, av, H, h, j0, p_i, m_use, mx, lsum, wp);
                l += lsum;
            }
            // W over the first half of U (the scores have all been read)
            tmem_st32(u_addr, *reinterpret_cast<uint32_t(*)[32]>(&wp[0]));
            tmem_st32(u_addr + 32u, *reinterpret_cast<uint32_t(*)[32]>(&wp[32]));
            tmem_st_wait();
            if (bl == 0 && t == n_tiles - 1 && j0 + KT > kv_len) {
                // keys at or past the valid length: clear their b^V rows so that
                // 0 * (whatever the cache holds there) stays 0 in the PV product
                uint8_t* bv = stage_bv(s);
                const int first = (kv_len - j0) * R;
                for (int rr = first + (threadIdx.x - 128); rr < 128; rr += 128)
                    for (int cb = 0; cb < NB; ++cb) {
                        uint4* pz = reinterpret_cast<uint4*>(bv + cb * kBox + rr * 128);
#pragma unroll
                        for (int e = 0; e < 8; ++e) pz[e] = make_uint4(0, 0, 0, 0);
                    }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            mbar_arrive(&w_ready[bl]);
        }
        const bool fin = alive && mbar_wait(&o_done[bl], 0u, lim, a.err, abort);
        if (__all_sync(0xffffffffu, fin)) {
            tc_fence_after();
            const float inv = a.out_scale / l;
            const long long t = (long long)b * a.S + q0 + i_loc;
            __nv_bfloat16* dst = a.out + (t * H + h) * DH;
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(lane_addr + o_col + (uint32_t)c * 32u, o);
                tmem_ld_wait();
                if (vq) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
                        *reinterpret_cast<uint4*>(dst + c * 32 + e) = w;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int DH, int R, int HC>
cudaError_t launch_t(const PrefillTcArgs& a0, const tpa_cache& c, int batch, const SeqParams& start,
                     cudaStream_t st) {
    PrefillTcArgs a = a0;
    constexpr int KT = 128 / R;
    constexpr int NB = DH / 64;
    a.a_bytes = (uint32_t)(KT * a.H * R * 2);
    const uint32_t a_pad = (a.a_bytes + 127u) & ~127u;
    a.stage_bytes = ((2u * NB * kBox + 2u * a_pad) + 1023u) & ~1023u;
    const uint32_t q_bytes = NB * 256u * 128u;
    const uint32_t budget = 227u * 1024u - 1024u - 256u - q_bytes;
    a.stages = std::min(4, (int)(budget / a.stage_bytes));
    if (a.stages < 2) return cudaErrorInvalidValue;
    CUtensorMap tmk, tmv;
    const uint64_t dims[2] = {(uint64_t)DH, (uint64_t)c.batch * c.capacity * R};
    const uint64_t stride[1] = {(uint64_t)DH * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_tmap_bf16(&tmk, c.b_k, 2, dims, stride, box) || !make_tmap_bf16(&tmv, c.b_v, 2, dims, stride, box))
        return cudaErrorInvalidValue;
    const size_t smem = 1024 + q_bytes + (size_t)a.stages * a.stage_bytes + (2 * a.stages + 7) * 8 + 16;
    cudaError_t e = allow_smem(reinterpret_cast<const void*>(prefill_tc_kernel<DH, R, HC>), (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_qblocks, batch);
    prefill_tc_kernel<DH, R, HC><<<grid, kThreads, smem, st>>>(tmk, tmv, a, start);
    return cudaGetLastError();
}
}  // namespace

bool prefill_tc_supported(const Shape& s) {
    if (!s.bf16) return false;
    if (s.Dh != 64 && s.Dh != 128) return false;
    if (s.Rk != s.Rv || (s.Rk != 1 && s.Rk != 2 && s.Rk != 4)) return false;
    if (s.H < 1 || 128 % s.H != 0) return false;
    if ((s.H * s.Rk) % 8 != 0) return false;          // 16-byte bulk copies of a^K / a^V rows
    if (s.Rq < 1 || s.Rq > 16) return false;
    return true;
}

cudaError_t launch_prefill_tc(const Shape& s, const tpa_factors& q, const tpa_cache& c, int batch,
                              int seqlen, const SeqParams& start, void* out, int* err,
                              uint32_t wait_limit, cudaStream_t st) {
    if ((long long)c.batch * c.capacity * s.Rk >= (1LL << 31)) return cudaErrorInvalidValue;
    PrefillTcArgs a{};
    a.a_q = static_cast<const __nv_bfloat16*>(q.a_q);
    a.b_q = static_cast<const __nv_bfloat16*>(q.b_q);
    a.ca_k = static_cast<const __nv_bfloat16*>(c.a_k);
    a.ca_v = static_cast<const __nv_bfloat16*>(c.a_v);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.S = seqlen;
    a.H = s.H;
    a.Rq = s.Rq;
    a.cap = c.capacity;
    a.qpb = 256 / s.H;
    a.n_qblocks = (seqlen + a.qpb - 1) / a.qpb;
    a.qscale = 1.4426950408889634f / ((float)s.Rq * (float)s.Rk * std::sqrt((float)s.Dh));
    a.out_scale = 1.f / (float)s.Rv;
    a.err = err;
    a.wait_limit = wait_limit;
    // head count 16 gets constant strides in the softmax loop; others read it at run time
    if (s.Dh == 64) {
        if (s.Rk == 2) return s.H == 16 ? launch_t<64, 2, 16>(a, c, batch, start, st)
                                        : launch_t<64, 2, 0>(a, c, batch, start, st);
        if (s.Rk == 1) return launch_t<64, 1, 0>(a, c, batch, start, st);
        return launch_t<64, 4, 0>(a, c, batch, start, st);
    }
    if (s.Rk == 2) return s.H == 16 ? launch_t<128, 2, 16>(a, c, batch, start, st)
                                    : launch_t<128, 2, 0>(a, c, batch, start, st);
    if (s.Rk == 1) return launch_t<128, 1, 0>(a, c, batch, start, st);
    return launch_t<128, 4, 0>(a, c, batch, start, st);
}

}  // namespace tpa
