// Causal prefill from the factor cache, query-major, on tcgen05 tensor cores (bf16
// operands, fp32 accumulate and softmax).
//
// The TPA attention of "【拜读】Tensor Product Attention Is All You Need…" (coreui.cn),
// §3 公式描述 and 代码 前向传播, evaluated from the cached factors (B_K already rotated,
// same page, 关键问题及回答 问题2); attention softmax(QK^T/sqrt(d_h))V per the jieyibu.net
// TPA page, Ⅱ.1.  K and V are formed tile by tile in shared memory and never reach
// device memory.
//
// One CTA takes 256 queries of one sequence (two query tiles of 128 rows) and a group
// of HG = 128/d_h heads.  The code is written for d_h 64 (HG 2) and 128 (HG 1), but only
// d_h 64 is dispatched here (see prefill_qm_supported).  Per key tile of 128 keys:
//   k_{j,h} = sum_s a^K_{j,h,s} b^K_{j,s},  v_{j,h} = sum_s a^V_{j,h,s} b^V_{j,s}
//             (bf16, formed once per tile for the group's heads, into shared memory)
// and then, per query tile w and head h of the group:
//   S      = q~_h . k_h^T      tcgen05, M = 128 queries, N = 128 keys, K = d_h
//   P      = 2^(S c - m)       online softmax (fp32), P as bf16 over S in TMEM
//   O_{w,h} += P . v_h         tcgen05, A = P from TMEM, B = v_h (MN-major)
//   out    = O / (l R_V)
// q~_h = sum_r a^Q_{i,h,r} b^Q_{i,r} (TPA; the query-side rank sum is done once per
// query) or the given rotated query (TPA-KVonly); c = log2(e) / (R_Q R_K sqrt(d_h))
// with R_Q = 1 for KV-only carries 1/R_Q, 1/R_K and the softmax scale.
//
// Warp roles (512 threads, one CTA per SM):
//   warp 0          the MMA issuer and TMEM owner: per step (key tile, head) PV(k) and
//                   QK(k+1) of query tile 0, then the same for tile 1 (warp 1 idles)
//   warps 2, 3      TMA producers, one staging slot each.  Copies issued by one thread
//                   complete one after another, so two producers with 32 KB boxes keep
//                   the staging ahead of the expander.
//   warps 4-7, 8-11 softmax of query tile 0 and 1, one query row per thread.  First they
//                   fold the queries: b^Q arrives one rank (and 64-column block) at a
//                   time through the staging slots, a^Q as one box, and each thread sums
//                   its row's a^Q_{h,r} b^Q_r in fp32 (KV-only: the query tiles arrive
//                   by TMA as they are)
//   warps 12-15     expander: staged b/a factor parts -> k_h, v_h tiles (swizzled)
// The issuer and the producers are the lowest-numbered warps: the warp schedulers favour
// them over the always-ready softmax warps of their sub-partitions, and the issuer's few
// instructions gate the tensor pipe.
// TMEM (512 columns): S_w at 256w (128 fp32 columns; P overwrites its first 64 as bf16
// pairs), O_{w,g} at 256w + 128 + g d_h.
// Shared basis (B_K, B_V shared across tokens, same page, 优点与创新 5): the b^K, b^V
// parts come from the layer's per-position tables (row = key position, for every
// sequence); nothing else changes.
#include <algorithm>
#include <cmath>

#include "tpa_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace tpa {

namespace {
using namespace sm100;

constexpr int kQmThreads = 512;
constexpr uint32_t kTile = 16384;                 // one [128 rows][128 B] swizzled block
constexpr uint32_t kPartMax = 32768;              // b bytes of one staged part
constexpr uint32_t kSlotBytes = kPartMax + 2048;  // + its a rows (16 B per key)
constexpr uint32_t kQOff = 0;                     // q~ [w][HG][NB] blocks: 64 KB
constexpr uint32_t kKOff = 65536;                 // k_h [HG][NB] blocks: 32 KB
constexpr uint32_t kVOff = 98304;                 // v_h [HG][NB] blocks: 32 KB
constexpr uint32_t kSlotOff = 131072;             // two staging slots
constexpr uint32_t kBarOff = kSlotOff + 2 * kSlotBytes;
constexpr int kNumBars = 29;                      // 27 barriers, TMEM address, abort flag
constexpr float kRescaleQm = 8.f;                 // lazy rescale threshold (log2 units)
// register split after the prologue: 256 softmax threads x 176 + 128 expander threads x
// 88 + 128 control threads x 56 = 63488 <= 512 threads x 128 at launch
constexpr int kRegSoftmaxQm = 176, kRegExpandQm = 88, kRegCtlQm = 56;

struct QmArgs {
    const __nv_bfloat16* a_q;     // [T][H][Rq] (TPA)
    const __nv_bfloat16* b_q;     // [T][Rq][D] (TPA) or the query [T][H][D] (KV-only)
    __nv_bfloat16* out;           // [T][H][D]
    int S, H, Rq, cap, bcap, batch, n_qblocks, n_groups;
    int n_fold;                   // staged b^Q slices per CTA: R_Q x (d_h / 64), 0 for KV-only
    int aw;                       // a^Q columns per staged row (a 16-byte multiple)
    int cache_batch;              // sequences the cache holds (bounds checks)
    long long T;                  // query rows (bounds checks)
    float sc;                     // log2(e) / (R_Q R_K sqrt(D))
    float out_scale;              // 1 / R_V
    int* err;
    uint32_t wait_limit;
};

template <int D, int R>
struct QmCfg {
    static constexpr int NB = D / 64;                        // 64-column blocks of d_h
    static constexpr int HG = 128 / D;                       // heads per CTA
    static constexpr int KP0 = (int)(kPartMax / (uint32_t)(R * D * 2));
    static constexpr int KP = KP0 < 128 ? KP0 : 128;         // keys per staged part
    static constexpr int PP = 128 / KP;                      // parts per K (or V) tile
    static constexpr uint32_t BBYTES = (uint32_t)KP * R * NB * 128;
    static constexpr uint32_t ABYTES = (uint32_t)KP * 16;
    static constexpr int TPK = 128 / KP;                     // expander threads per key
    static constexpr int CPT = NB * 8 / TPK;                 // 16-byte chunks per thread
    static_assert(HG * R <= 8, "a-factor box holds 8 values per key");
    static_assert(KP * TPK == 128 && CPT * TPK == NB * 8, "expander split");
};

// bf16 element `idx` (0..7) of a 16-byte row, broadcast to both halves of a bf16x2
__device__ __forceinline__ uint32_t bcast_bf16(const uint4& v, int idx) {
    const uint32_t w = idx < 4 ? (idx < 2 ? v.x : v.y) : (idx < 6 ? v.z : v.w);
    const uint32_t h = (idx & 1) ? (w >> 16) : (w & 0xffffu);
    return h | (h << 16);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// 2^d for a pair of exponents on the FMA pipe, beside ex2.approx on MUFU (Cody–Waite style
// range reduction with a fitted polynomial): d = n + f with n = round(d) -- adding 1.5 * 2^23
// leaves n in the low mantissa bits -- and f in [-1/2, 1/2]; 2^f by a cubic whose
// coefficients were fitted by Remez exchange to equioscillating relative error on
// [-1/2, 1/2] (7.5e-5, evaluated in fp32 Horner form, against the 2^-9 half-ulp of the
// bf16 P); n is then added to the exponent field.  d is clamped at -126 so that the
// exponent field stays in range (such terms give at most 2^-126).
constexpr float kE2C0 = 0.99992806f, kE2C1 = 0.69326097f, kE2C2 = 0.24261113f, kE2C3 = 0.05517167f;
// Key pairs of a 32-column chunk whose exp2 runs on the FMA pipe: every kFmaExpEvery-th pair
// (0: none).  Measured at b8 x s2048 with every 4th pair: 0.2395 ms against 0.2316 ms with
// all of them on MUFU.  MUFU is not this kernel's bound (31% busy); the split's extra FMA
// and integer instructions cost more issue slots than the MUFU time they save.
constexpr int kFmaExpEvery = 0;
[[maybe_unused]] constexpr int kFmaExpMod = kFmaExpEvery > 0 ? kFmaExpEvery : 1;
[[maybe_unused]] __device__ __forceinline__ void ex2_fma_pair(float d0, float d1, float& p0, float& p1) {
    constexpr float kShift = 12582912.f;   // 1.5 * 2^23
    const uint64_t dd = pk2(fmaxf(d0, -126.f), fmaxf(d1, -126.f));
    const uint64_t t = fadd2(dd, pk2(kShift, kShift));
    const uint64_t n = fadd2(t, pk2(-kShift, -kShift));
    const uint64_t f = ffma2(n, pk2(-1.f, -1.f), dd);
    uint64_t q = ffma2(f, pk2(kE2C3, kE2C3), pk2(kE2C2, kE2C2));
    q = ffma2(q, f, pk2(kE2C1, kE2C1));
    q = ffma2(q, f, pk2(kE2C0, kE2C0));
    float t0, t1, q0, q1;
    upk2(t, t0, t1);
    upk2(q, q0, q1);
    p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

template <int D, int R>
__global__ void __launch_bounds__(kQmThreads, 1)
prefill_qm_kernel(const __grid_constant__ CUtensorMap tbk, const __grid_constant__ CUtensorMap tbv,
                  const __grid_constant__ CUtensorMap tak, const __grid_constant__ CUtensorMap tav,
                  const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap taq,
                  const QmArgs a, const SeqParams start) {
    using C = QmCfg<D, R>;
    constexpr int NB = C::NB, HG = C::HG, KP = C::KP, PP = C::PP;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
    uint64_t* slot_full = bars;          // [2] a staged part has landed
    uint64_t* slot_empty = bars + 2;     // [2] the expander has read it
    uint64_t* q_full = bars + 4;         // [1] q~ of both query tiles is in shared memory
    uint64_t* kx_full = bars + 5;        // [HG] k_g of the current tile is written
    uint64_t* vx_full = bars + 7;        // [HG] v_g ...
    uint64_t* kx_empty = bars + 9;       // [2 w][HG] QK(w, g) of the tile has completed
    uint64_t* vx_empty = bars + 13;      // [2 w][HG] PV(w, g) ...
    uint64_t* s_full = bars + 17;        // [2] scores of query tile w are in TMEM
    // bars + 19, 20: unused
    uint64_t* o_done = bars + 21;        // [2] the last PV of query tile w has completed
    uint64_t* fin = bars + 23;           // [2] each issuer's MMAs in flight at exit
    uint64_t* a_full = bars + 25;        // [1] a^Q (KV-only: the query tiles) has landed
    uint64_t* pp_go = bars + 26;         // [1] query tile 0's first P is done: tile 1 may start
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 27);
    volatile int* abort = reinterpret_cast<volatile int*>(bars + 28);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lim = a.wait_limit;

    // ---- the work unit: longest query blocks first
    const int per_qb = a.n_groups * a.batch;
    const int qb = a.n_qblocks - 1 - (int)blockIdx.x / per_qb;
    const int rem = (int)blockIdx.x % per_qb;
    const int b = rem / a.n_groups;
    const int g0 = (rem % a.n_groups) * HG;
    const int q0 = qb * 256;
    const int st0 = start.v[b];
    const int kv_len = st0 + a.S;
    // key tiles each query tile needs (0 for a tile past the sequence's end)
    const int n_w0 = (st0 + min(q0 + 127, a.S - 1)) / 128 + 1;
    const int n_w1 = q0 + 128 < a.S ? (st0 + min(q0 + 255, a.S - 1)) / 128 + 1 : 0;
    auto n_w = [&](int w) { return w ? n_w1 : n_w0; };
    const int n_max = max(n_w0, n_w1);
    const int xa = (g0 * R) / 8 * 8;      // first a-factor column of the staged box
    const int xq = (g0 * a.Rq) / 8 * 8;   // first a^Q column of the staged query box
    const long long t0 = (long long)b * a.S + q0;   // the CTA's first query token

    if (threadIdx.x == 0) {
        // arrivals per phase: commits and producer arrivals 1; expander warps 4; softmax
        // warps 4 per query tile, 8 for q_full; slot_empty 8 (the 8 softmax warps after a
        // b^Q slice, or the 4 expander warps counting 2 each after a factor part)
        for (int s = 0; s < 2; ++s) { mbar_init(&slot_full[s], 1); mbar_init(&slot_empty[s], 8); }
        mbar_init(q_full, 8);
        mbar_init(a_full, 1);
        mbar_init(pp_go, 1);
        for (int g = 0; g < 2; ++g) { mbar_init(&kx_full[g], 4); mbar_init(&vx_full[g], 4); }
        for (int i = 0; i < 4; ++i) { mbar_init(&kx_empty[i], 1); mbar_init(&vx_empty[i], 1); }
        for (int w = 0; w < 2; ++w) {
            mbar_init(&s_full[w], 1);
            mbar_init(&o_done[w], 1); mbar_init(&fin[w], 1);
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == 2 && lane == 0) {
        prefetch_tensormap(&tbk); prefetch_tensormap(&tbv);
        prefetch_tensormap(&tak); prefetch_tensormap(&tav);
        prefetch_tensormap(&tq); prefetch_tensormap(&taq);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 4 && warp < 12) {
        // ================================================================ softmax
        const int w = (warp - 4) >> 2;
        const int r = (warp & 3) * 32 + lane;
        const int i = q0 + 128 * w + r;
        const bool vq = i < a.S;
        const long long t = (long long)b * a.S + i;
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmaxQm));
        // ---- fold the query: q~ rows of the group's heads, swizzled, into shared memory
        {
            const int rc = 128 * w + r;                   // row within the CTA's 256 queries
            bool fok = mbar_wait(a_full, 0u, lim, a.err, abort);
            if (a.Rq > 0) {
                // a^Q rows sit at the start of the q~ area until every thread has read them
                const uint32_t arow = smem_u32(smem + kQOff) + (uint32_t)(rc * a.aw * 2);
                float acc[HG][D];
#pragma unroll
                for (int g = 0; g < HG; ++g)
#pragma unroll
                    for (int e = 0; e < D; ++e) acc[g][e] = 0.f;
                for (int n = 0; n < a.n_fold; ++n) {
                    const int slot = n & 1;
                    fok = fok && mbar_wait(&slot_full[slot], (uint32_t)((n >> 1) & 1), lim, a.err, abort);
                    const int rq = n / NB, hf = n % NB;   // rank, and the half of the rows (d_h 128)
                    if (fok && (NB == 1 || hf == w)) {
                        const uint32_t src = smem_u32(smem + kSlotOff + (uint32_t)slot * kSlotBytes);
                        const uint32_t row = (uint32_t)(NB == 1 ? rc : r);
                        float av[HG];
#pragma unroll
                        for (int g = 0; g < HG; ++g)
                            av[g] = __uint_as_float(lds_u16(arow + (uint32_t)(((g0 + g) * a.Rq + rq - xq) * 2)) << 16);
#pragma unroll
                        for (int cb = 0; cb < NB; ++cb)
#pragma unroll
                            for (int c8 = 0; c8 < 8; ++c8) {
                                // consecutive rows sit in different swizzle phases: the
                                // threads of a quarter-warp read different banks
                                const uint4 v = lds_v4(src + sw128_offset(row * NB + (uint32_t)cb, (uint32_t)c8 * 16u));
                                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float lo = bf16lo(wv[e]), hi = bf16hi(wv[e]);
#pragma unroll
                                    for (int g = 0; g < HG; ++g) {
                                        acc[g][cb * 64 + c8 * 8 + 2 * e] = fmaf(av[g], lo, acc[g][cb * 64 + c8 * 8 + 2 * e]);
                                        acc[g][cb * 64 + c8 * 8 + 2 * e + 1] = fmaf(av[g], hi, acc[g][cb * 64 + c8 * 8 + 2 * e + 1]);
                                    }
                                }
                            }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&slot_empty[slot]);
                }
                bar_sync(1, 256);                         // every a^Q row has been read
#pragma unroll
                for (int g = 0; g < HG; ++g)
#pragma unroll
                    for (int c = 0; c < NB * 8; ++c) {
                        uint8_t* dst = smem + kQOff + (uint32_t)((w * 2 + g * NB) + c / 8) * kTile +
                                       sw128_offset((uint32_t)r, (uint32_t)(c % 8) * 16u);
                        *reinterpret_cast<uint4*>(dst) =
                            make_uint4(pack_bf16(acc[g][8 * c], acc[g][8 * c + 1]), pack_bf16(acc[g][8 * c + 2], acc[g][8 * c + 3]),
                                       pack_bf16(acc[g][8 * c + 4], acc[g][8 * c + 5]), pack_bf16(acc[g][8 * c + 6], acc[g][8 * c + 7]));
                    }
                fence_proxy_async_smem();
            }
            (void)fok;
            __syncwarp();
            if (lane == 0) mbar_arrive(q_full);
        }

        const int nt = n_w(w);
        const int p_i = st0 + i;                       // this row's position
        const int p_first = st0 + q0 + 128 * w;        // the tile's first row
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t s_addr = lane_base + 256u * (uint32_t)w;
        // running max (scaled, log2 units) and sum of each head of the group
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        const float sc = a.sc;
        const uint64_t sc2 = pk2(sc, sc);
        bool alive = true;
        // ---- this query tile's MMAs, issued by one thread of the group (the leader)
        // once the group's P is in TMEM: PV(k), then QK(k+1) into the same S columns
        // (in order, so QK(k+1) writes S only after PV(k) has read P).  Descriptors are
        // formed once: stepping K by 16 adds 32 bytes, i.e. 2 in the descriptor's address
        // field (address / 16, no carry below 256 KB); 64-column blocks are kTile apart.
        const bool leader = (warp & 3) == 0 && lane == 0;
        const int K = nt * HG;                         // steps (key tile, head)
        const uint32_t s_col = tmem + 256u * (uint32_t)w;
        const uint32_t idesc_qk = idesc_bf16(128, 128, 0, 0);
        const uint32_t idesc_pv = idesc_bf16(128, D, 0, 1);
        const uint64_t qd0 = smem_desc(smem_u32(smem + kQOff + (uint32_t)(w * 2) * kTile), 16, 1024, kSwizzle128);
        const uint64_t qd1 = smem_desc(smem_u32(smem + kQOff + (uint32_t)(w * 2 + (HG - 1) * NB) * kTile), 16, 1024, kSwizzle128);
        const uint64_t kd0 = smem_desc(smem_u32(smem + kKOff), 16, 1024, kSwizzle128);
        const uint64_t kd1 = smem_desc(smem_u32(smem + kKOff + (uint32_t)((HG - 1) * NB) * kTile), 16, 1024, kSwizzle128);
        const uint64_t vd0 = smem_desc(smem_u32(smem + kVOff), kTile, 1024, kSwizzle128);
        const uint64_t vd1 = smem_desc(smem_u32(smem + kVOff + (uint32_t)((HG - 1) * NB) * kTile), kTile, 1024, kSwizzle128);
        auto issue_qk = [&](int kq) {
            const int gq = HG == 1 ? 0 : kq % HG;
            const uint64_t qa = gq ? qd1 : qd0, kb = gq ? kd1 : kd0;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t off = (uint64_t)((kk >> 2) * (kTile >> 4) + (kk & 3) * 2);
                mma_ss(s_col, qa + off, kb + off, idesc_qk, kk > 0 ? 1u : 0u);
            }
            mma_commit(&s_full[w]);
            mma_commit(&kx_empty[w * HG + gq]);
        };
        auto issue_pv = [&](int kp, bool last) {
            const int jp = kp / HG, gp = HG == 1 ? 0 : kp % HG;
            const uint64_t vb = gp ? vd1 : vd0;
            const uint32_t o_col = s_col + 128u + (uint32_t)(gp * D);
            mma_ts(o_col, s_col, vb, idesc_pv, jp > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 1; kk < 8; ++kk)
                mma_ts(o_col, s_col + (uint32_t)kk * 8u, vb + (uint64_t)(kk * 128), idesc_pv, 1u);
            mma_commit(&vx_empty[w * HG + gp]);
            if (last) mma_commit(&o_done[w]);
        };
        int vs = -1, ks = 0;       // steps whose v (k) tiles are known written: <= vs (<= ks)
        if (leader && K > 0) {
            // tile 1 starts one softmax behind tile 0, so that one tile's MMAs run while
            // the other's softmax works (pp_go has one phase: the wait cannot alias)
            bool ok = mbar_wait(q_full, 0u, lim, a.err, abort) && mbar_wait(&kx_full[0], 0u, lim, a.err, abort);
            if (ok && w == 1) ok = mbar_wait(pp_go, 0u, lim, a.err, abort);
            if (ok) {
                tc_fence_after();
                issue_qk(0);
            }
        }
        __syncwarp();        // the leader's warp reconverges before the aligned barriers below
        // One rolled step per (key tile, head): the step's code stays small.
#pragma unroll 1
        for (int k = 0; k < nt * HG; ++k) {
            const int j = k / HG, g = k % HG;
            const bool okw = mbar_wait(&s_full[w], (uint32_t)(k & 1), lim, a.err, abort);
            // the group's 128 threads vote, so they all leave together if a wait gave up
            // (the step's second barrier below is then reached by all or by none)
            if (bar_any(2 + w, 128, !okw)) { alive = false; break; }
            tc_fence_after();
            const int j0 = j * 128;
            const bool masked = j0 + 127 > p_first;
            const int lim_c = p_i - j0;                // key j0 + c is visible iff c <= lim_c
            // ---- pass 1: the tile's max, two 32-column chunks per TMEM wait
            uint32_t sa[32], sb[32];
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                tmem_ld32(s_addr + 64u * (uint32_t)h, sa);
                tmem_ld32(s_addr + 64u * (uint32_t)h + 32u, sb);
                tmem_ld_wait();
                const int cb = 64 * h;
                if (masked) {
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        mx0 = fmax3(mx0, cb + c <= lim_c ? __uint_as_float(sa[c]) : -INFINITY,
                                    cb + c + 1 <= lim_c ? __uint_as_float(sa[c + 1]) : -INFINITY);
                        mx1 = fmax3(mx1, cb + 32 + c <= lim_c ? __uint_as_float(sb[c]) : -INFINITY,
                                    cb + 33 + c <= lim_c ? __uint_as_float(sb[c + 1]) : -INFINITY);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        mx0 = fmax3(mx0, __uint_as_float(sa[c]), __uint_as_float(sa[c + 1]));
                        mx1 = fmax3(mx1, __uint_as_float(sb[c]), __uint_as_float(sb[c + 1]));
                    }
                }
            }
            const float mxs = fmaxf(mx0, mx1) * sc;
            float mg = (HG == 1 || g == 0) ? m0 : m1;
            float lg = (HG == 1 || g == 0) ? l0 : l1;
            float alpha = 1.f;
            if (mxs > mg + kRescaleQm) {               // first tile, or the max rose by > 2^8
                alpha = ex2(mg - mxs);
                mg = mxs;
            }
            lg *= alpha;
            // ---- pass 2: p = 2^(s c - m), row sum, P over the first 64 columns of S
            const uint64_t negm2 = pk2(-mg, -mg);
            uint64_t sum2a = pk2(0.f, 0.f), sum2b = sum2a;
            auto exp_chunk = [&](const uint32_t (&sv)[32], int cb, uint32_t (&pk)[16]) {
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    float d0, d1;
                    upk2(ffma2(pk2(__uint_as_float(sv[2 * q]), __uint_as_float(sv[2 * q + 1])), sc2, negm2), d0, d1);
                    if (masked) {
                        d0 = cb + 2 * q <= lim_c ? d0 : -INFINITY;
                        d1 = cb + 2 * q + 1 <= lim_c ? d1 : -INFINITY;
                    }
                    float p0 = 0.f, p1 = 0.f;
                    bool on_mufu = true;
                    if constexpr (kFmaExpEvery > 0) {
                        if (q % kFmaExpMod == kFmaExpMod - 1) {
                            on_mufu = false;
                            ex2_fma_pair(d0, d1, p0, p1);
                            if (masked) {
                                p0 = cb + 2 * q <= lim_c ? p0 : 0.f;
                                p1 = cb + 2 * q + 1 <= lim_c ? p1 : 0.f;
                            }
                        }
                    }
                    if (on_mufu) {
                        p0 = ex2(d0);
                        p1 = ex2(d1);
                    }
                    if (q & 1) sum2b = fadd2(sum2b, pk2(p0, p1));
                    else sum2a = fadd2(sum2a, pk2(p0, p1));
                    pk[q] = pack_bf16(p0, p1);
                }
            };
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                // columns 64h.. of S are read before P of keys 64h.. lands on columns 32h..
                tmem_ld32(s_addr + 64u * (uint32_t)h, sa);
                tmem_ld32(s_addr + 64u * (uint32_t)h + 32u, sb);
                tmem_ld_wait();
                uint32_t pk[16];
                exp_chunk(sa, 64 * h, pk);
                tmem_st16(s_addr + 32u * (uint32_t)h, pk);
                exp_chunk(sb, 64 * h + 32, pk);
                tmem_st16(s_addr + 32u * (uint32_t)h + 16u, pk);
            }
            float sa0, sa1, sb0, sb1;
            upk2(sum2a, sa0, sa1);
            upk2(sum2b, sb0, sb1);
            lg += (sa0 + sa1) + (sb0 + sb1);
            if (HG == 1 || g == 0) { m0 = mg; l0 = lg; } else { m1 = mg; l1 = lg; }
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                // O_{w,g} row *= alpha: the PVs into it so far have completed (the
                // scores of this step were committed after them)
                const uint32_t o_addr = lane_base + 256u * (uint32_t)w + 128u + (uint32_t)(g * D);
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    tmem_ld32(o_addr + 32u * c, sa);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) sa[e] = __float_as_uint(__uint_as_float(sa[e]) * alpha);
                    tmem_st32(o_addr + 32u * c, sa);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            bar_sync(2 + w, 128);                      // the group's P (and O) is in TMEM
            if (leader) {
                // tile 1 may start now; released before the waits below, one of which
                // (the next key tile) needs tile 1's first QK to have completed
                if (w == 0 && k == 0) mbar_arrive(pp_go);
                // The expander writes k_0, .., k_{HG-1}, v_0, .., v_{HG-1} of a tile, then
                // the next tile's, in that order, so one wait covers both tiles a step
                // needs: v_g of tile j for PV(k), and k of step k+1, which is written
                // before v_g unless step k+1 starts the next tile (then after it).
                const bool more = k + 1 < K;
                const int k1 = k + 1;
                const bool newtile = more && k1 % HG == 0;
                bool ok = true;
                if (newtile ? ks < k1 : vs < k) {
                    if (newtile) {
                        ok = mbar_wait(&kx_full[0], (uint32_t)((k1 / HG) & 1), lim, a.err, abort);
                        ks = k1;
                        vs = k;
                    } else {
                        ok = mbar_wait(&vx_full[g], (uint32_t)(j & 1), lim, a.err, abort);
                        vs = k;
                        ks = max(ks, j * HG + HG - 1);
                    }
                }
                if (ok) {
                    tc_fence_after();
                    issue_pv(k, !more);
                    if (more) issue_qk(k + 1);
                }
            }
            __syncwarp();    // reconverge: the next step's barrier vote is warp-aligned
        }
        if (leader) {
            // every MMA this thread issued completes before TMEM is released
            mma_commit(&fin[w]);
            drain_wait(&fin[w], 0u);
        }
        if (nt > 0) {
            const bool done_ok = alive && mbar_wait(&o_done[w], 0u, lim, a.err, abort);
            if (__all_sync(0xffffffffu, done_ok)) {
                tc_fence_after();
#pragma unroll
                for (int g = 0; g < HG; ++g) {
                    const float inv = a.out_scale / ((HG == 1 || g == 0) ? l0 : l1);
                    const uint32_t o_addr = lane_base + 256u * (uint32_t)w + 128u + (uint32_t)(g * D);
                    __nv_bfloat16* dst = a.out + (t * a.H + g0 + g) * D;
                    const bool st_ok = vq && in_bounds(t < a.T, a.err);
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + 32u * c, o);
                        tmem_ld_wait();
                        if (st_ok) {
#pragma unroll
                            for (int e = 0; e < 32; e += 8) {
                                uint4 v;
                                v.x = pack_bf16(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
                                v.y = pack_bf16(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
                                v.z = pack_bf16(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
                                v.w = pack_bf16(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
                                *reinterpret_cast<uint4*>(dst + c * 32 + e) = v;
                            }
                        }
                    }
                }
            }
        }
    } else if (warp >= 12) {
        // ================================================================ expander
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegExpandQm));
        const int e = threadIdx.x - 384;
        const int kl = e % KP;                       // key within a part
        const int c0 = (e / KP) * C::CPT;            // first 16-byte chunk of the row
        int n = a.n_fold;                            // slot phases (the b^Q slices come first)
        // The slots carry the b^Q slices first.  A parity wait only tells the current
        // phase from the one before it, so the expander must not poll a slot until the
        // fold has consumed every slice: then each slot's next phase is this part's.
        bool ok = a.n_fold == 0 || mbar_wait(q_full, 0u, lim, a.err, abort);
        for (int j = 0; j < n_max && ok; ++j) {
            for (int p = 0; p < 2 * PP; ++p, ++n) {
                const int slot = n & 1;
                if (!mbar_wait(&slot_full[slot], (uint32_t)((n >> 1) & 1), lim, a.err, abort)) { ok = false; break; }
                const bool isK = p < PP;
                const int pp = isK ? p : p - PP;
                const uint8_t* src = smem + kSlotOff + (uint32_t)slot * kSlotBytes;
                const uint32_t src_u = smem_u32(src);
                const uint4 araw = lds_v4(src_u + kPartMax + (uint32_t)kl * 16u);
                const int key = j * 128 + pp * KP + kl;
                const bool valid = key < kv_len;
                const uint32_t row_out = (uint32_t)(pp * KP + kl);

#pragma unroll
                for (int g = 0; g < HG; ++g) {
                    // k_g (v_g) of tile j-1 is free once the QKs (PVs) of both query tiles
                    // that read it have completed; the other head's buffer may still be busy.
                    // These barriers have one phase per tile, and the next phase needs the
                    // tile written here, so a parity wait cannot be overtaken.
                    if (pp == 0 && j >= 1) {
                        uint64_t* empty = isK ? kx_empty : vx_empty;
#pragma unroll
                        for (int w = 0; w < 2; ++w)
                            if (j - 1 < n_w(w) &&
                                !mbar_wait(&empty[w * HG + g], (uint32_t)((j - 1) & 1), lim, a.err, abort))
                                ok = false;
                    }
                    if (!ok) break;
                    // k = sum_s a_s b_s for this key and head, accumulated in fp32 (packed
                    // pairs) and rounded to bf16 once: bf16 products and sums would round at
                    // every rank, which costs a visible part of the error budget
                    uint8_t* dst0 = smem + (isK ? kKOff : kVOff) + (uint32_t)(g * NB) * kTile;
                    uint64_t af[R];
#pragma unroll
                    for (int s2 = 0; s2 < R; ++s2) {
                        const float av = __uint_as_float(bcast_bf16(araw, (g0 + g) * R + s2 - xa) << 16);
                        af[s2] = pk2(av, av);
                    }
#pragma unroll 4
                    for (int cc = 0; cc < C::CPT; ++cc) {
                        const int c = c0 + cc;
                        const int cb = c / 8, c8 = c % 8;
                        uint64_t acc[4];
#pragma unroll
                        for (int s2 = 0; s2 < R; ++s2) {
                            const uint4 bv = lds_v4(src_u + sw128_offset((uint32_t)((kl * R + s2) * NB + cb), (uint32_t)c8 * 16u));
                            const uint32_t wv[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                acc[e] = ffma2(pk2(bf16lo(wv[e]), bf16hi(wv[e])), af[s2], s2 == 0 ? pk2(0.f, 0.f) : acc[e]);
                        }
                        uint32_t ow[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float lo, hi;
                            upk2(acc[e], lo, hi);
                            ow[e] = pack_bf16(lo, hi);
                        }
                        uint4 o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                        if (!valid) o = make_uint4(0, 0, 0, 0);  // keys past the cached length
                        *reinterpret_cast<uint4*>(dst0 + (uint32_t)cb * kTile + sw128_offset(row_out, (uint32_t)c8 * 16u)) = o;
                    }
                    if (pp == PP - 1) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(isK ? &kx_full[g] : &vx_full[g]);
                    }
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) mbar_arrive_cnt(&slot_empty[slot], 2);
            }
        }
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegCtlQm));
        if (warp < 2) {
            // warp 0 owns the TMEM (allocated above, released below); warps 0 and 1 idle
        } else {
            // ============================================================ producers
            const int pid = warp - 2;                   // slot pid: items pid, pid + 2, ...
            if (lane == 0) {
                if (pid == 0) {
                    // the queries: a^Q rows of the group (TPA), or the query tiles (KV-only)
                    if (a.Rq > 0) {
                        mbar_arrive_expect_tx(a_full, (uint32_t)(a.aw * 2 * 256));
                        tma_load_2d(smem + kQOff, &taq, a_full, xq, (int)t0);
                    } else {
                        mbar_arrive_expect_tx(a_full, 2u * HG * NB * kTile);
#pragma unroll
                        for (int w = 0; w < 2; ++w)
#pragma unroll
                            for (int g = 0; g < HG; ++g)
#pragma unroll
                                for (int cb = 0; cb < NB; ++cb)
                                    tma_load_4d(smem + kQOff + (uint32_t)((w * 2 + g * NB) + cb) * kTile, &tq, a_full,
                                                0, cb, g0 + g, (int)t0 + 128 * w);
                    }
                }
                const int n_items = a.n_fold + n_max * 2 * PP;
                const int brow0 = a.bcap ? b * a.bcap : 0;
                const int arow0 = b * a.cap;
                int u = 0;                              // fills of this slot
                for (int n = pid; n < n_items && !*abort; n += 2, ++u) {
                    if (u >= 1 && !mbar_wait(&slot_empty[pid], (uint32_t)((u - 1) & 1), lim, a.err, abort)) break;
                    uint8_t* dst = smem + kSlotOff + (uint32_t)pid * kSlotBytes;
                    if (n < a.n_fold) {
                        // b^Q of rank n / NB for the CTA's rows (all 256, or half n % NB at d_h 128)
                        mbar_arrive_expect_tx(&slot_full[pid], kPartMax);
                        tma_load_4d(dst, &tq, &slot_full[pid], 0, 0, n / NB, (int)t0 + (n % NB) * (256 / NB));
                        continue;
                    }
                    const int m = n - a.n_fold;
                    const int j = m / (2 * PP), p = m % (2 * PP);
                    const bool isK = p < PP;
                    const int key0 = j * 128 + (isK ? p : p - PP) * KP;
                    mbar_arrive_expect_tx(&slot_full[pid], C::BBYTES + C::ABYTES);
                    tma_load_4d(dst, isK ? &tbk : &tbv, &slot_full[pid], 0, 0, 0, brow0 + key0);
                    tma_load_2d(dst + kPartMax, isK ? &tak : &tav, &slot_full[pid], xa, arow0 + key0);
                }
                if (pid == 0) drain_wait(a_full, 0u);
                if (u > 0) drain_wait(&slot_full[pid], (uint32_t)((u - 1) & 1));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, int R>
cudaError_t launch_qm(const QmArgs& a, const tpa_cache& c, const SeqParams& start, cudaStream_t st) {
    using C = QmCfg<D, R>;
    CUtensorMap tbk, tbv, tak, tav;
    // B rows: every sequence's (contextual), or one per-position table (shared basis);
    // the box lands as [key][rank][d_h block][64], 128-byte rows, swizzled
    const uint64_t b_rows = (uint64_t)(a.bcap ? c.batch : 1) * (uint64_t)c.capacity;
    const uint64_t bd[4] = {64, (uint64_t)C::NB, (uint64_t)R, b_rows};
    const uint64_t bs[3] = {128, (uint64_t)D * 2, (uint64_t)R * D * 2};
    const uint32_t bb[4] = {64, (uint32_t)C::NB, (uint32_t)R, (uint32_t)C::KP};
    if (!make_tmap_bf16(&tbk, c.b_k, 4, bd, bs, bb) || !make_tmap_bf16(&tbv, c.b_v, 4, bd, bs, bb))
        return cudaErrorInvalidValue;
    // A rows of every sequence: a box of 8 values (16 bytes) per key around the group's heads
    const uint64_t ad[2] = {(uint64_t)a.H * R, (uint64_t)c.batch * (uint64_t)c.capacity};
    const uint64_t as[1] = {(uint64_t)a.H * R * 2};
    const uint32_t ab[2] = {8, (uint32_t)C::KP};
    if (!make_tmap_bf16(&tak, c.a_k, 2, ad, as, ab, 0) || !make_tmap_bf16(&tav, c.a_v, 2, ad, as, ab, 0))
        return cudaErrorInvalidValue;
    // queries: b^Q [T][R_Q][d_h] as [64][block][rank][token] with boxes of one rank and
    // 256 / NB tokens (32 KB, one staging slot); KV-only: q [T][h][d_h] with boxes of one
    // 64-column block of one head for 128 tokens (one q~ block); a^Q [T][h R_Q] rows
    CUtensorMap tq, taq;
    if (a.Rq > 0) {
        const uint64_t qd[4] = {64, (uint64_t)C::NB, (uint64_t)a.Rq, (uint64_t)a.T};
        const uint64_t qs[3] = {128, (uint64_t)D * 2, (uint64_t)a.Rq * D * 2};
        const uint32_t qb[4] = {64, (uint32_t)C::NB, 1, (uint32_t)(256 / C::NB)};
        const uint64_t aqd[2] = {(uint64_t)a.H * a.Rq, (uint64_t)a.T};
        const uint64_t aqs[1] = {(uint64_t)a.H * a.Rq * 2};
        const uint32_t aqb[2] = {(uint32_t)a.aw, 256};
        if (!make_tmap_bf16(&tq, a.b_q, 4, qd, qs, qb) || !make_tmap_bf16(&taq, a.a_q, 2, aqd, aqs, aqb, 0))
            return cudaErrorInvalidValue;
    } else {
        const uint64_t qd[4] = {64, (uint64_t)C::NB, (uint64_t)a.H, (uint64_t)a.T};
        const uint64_t qs[3] = {128, (uint64_t)D * 2, (uint64_t)a.H * D * 2};
        const uint32_t qb[4] = {64, 1, 1, 128};
        if (!make_tmap_bf16(&tq, a.b_q, 4, qd, qs, qb)) return cudaErrorInvalidValue;
        taq = tq;
    }
    const size_t smem = 1024 + kBarOff + kNumBars * 8;
    cudaError_t e = allow_smem(reinterpret_cast<const void*>(prefill_qm_kernel<D, R>), (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)a.n_qblocks * a.n_groups * a.batch;
    if (grid < 1 || grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    prefill_qm_kernel<D, R><<<(unsigned)grid, kQmThreads, smem, st>>>(tbk, tbv, tak, tav, tq, taq, a, start);
    return cudaGetLastError();
}

}  // namespace

// a^Q columns the staged box must span so that every head group's h_g R_Q values fit,
// from the 16-byte-aligned column below the group's first one
static int qm_a_width(const Shape& s) {
    const int hg = 128 / s.Dh;
    int need = 0;
    for (int g0 = 0; g0 < s.H; g0 += hg) {
        const int x0 = (g0 * s.Rq) / 8 * 8;
        need = std::max(need, (g0 + hg) * s.Rq - x0);
    }
    return (need + 7) / 8 * 8;
}

bool prefill_qm_supported(const Shape& s) {
    if (!s.bf16) return false;
    // d_h 64 only.  At d_h 128 a CTA holds one head (the two query tiles' O fill the
    // TMEM), so every head re-stages and re-expands the key tiles and the kernel is
    // bound by shared-memory traffic: measured 2.82 ms against 2.31 ms for the
    // (query, head)-row kernel on the b4 x s8192, h 16 layer, which therefore takes it.
    if (s.Dh != 64) return false;
    if (s.Rk != s.Rv || (s.Rk != 1 && s.Rk != 2 && s.Rk != 4)) return false;
    const int hg = 128 / s.Dh;
    if (s.H < hg || s.H % hg != 0) return false;
    if ((s.H * s.Rk) % 8 != 0) return false;     // 16-byte rows of the a-factor maps
    if (hg * s.Rk > 8) return false;             // the group's a values fit one 16-byte box
    if (s.Rq < 0 || s.Rq > 16) return false;     // 0: TPA-KVonly, the query is given
    if (s.Rq > 0 && (s.H * s.Rq) % 8 != 0) return false;   // 16-byte rows of the a^Q map
    if (s.Rq > 0 && qm_a_width(s) > 128) return false;    // the a^Q box (256 rows) fits the q~ area
    return true;
}

cudaError_t launch_prefill_qm(const Shape& s, const tpa_factors& q, const tpa_cache& c, int batch,
                              int seqlen, const SeqParams& start, void* out, int* err,
                              uint32_t wait_limit, cudaStream_t st) {
    if ((long long)c.batch * c.capacity >= (1LL << 31)) return cudaErrorInvalidValue;
    QmArgs a{};
    a.a_q = static_cast<const __nv_bfloat16*>(q.a_q);
    a.b_q = static_cast<const __nv_bfloat16*>(q.b_q);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.S = seqlen;
    a.H = s.H;
    a.Rq = s.Rq;
    a.cap = c.capacity;
    a.bcap = (int)b_seq_rows(s, c);
    a.batch = batch;
    a.n_qblocks = (seqlen + 255) / 256;
    a.n_groups = s.H / (128 / s.Dh);
    a.n_fold = s.Rq > 0 ? s.Rq * (s.Dh / 64) : 0;
    a.aw = s.Rq > 0 ? qm_a_width(s) : 0;
    a.cache_batch = c.batch;
    a.T = (long long)batch * seqlen;
    a.sc = 1.4426950408889634f / ((float)(s.Rq > 0 ? s.Rq : 1) * (float)s.Rk * std::sqrt((float)s.Dh));
    a.out_scale = 1.f / (float)s.Rv;
    a.err = err;
    a.wait_limit = wait_limit;
    if (s.Dh != 64) return cudaErrorInvalidValue;
    if (s.Rk == 2) return launch_qm<64, 2>(a, c, start, st);
    if (s.Rk == 1) return launch_qm<64, 1>(a, c, start, st);
    return launch_qm<64, 4>(a, c, start, st);
}

}  // namespace tpa
