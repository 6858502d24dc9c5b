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
// walking key tiles of KT = 64/R keys (64 U columns).  Warp roles:
//   warp 0     TMA: b^K, b^V tiles (2-D maps over the cache, 128-byte swizzle) and
//              a^K, a^V tiles (bulk copies) into a ring of stages
//   warps 1-2  MMA issuers, one per M-block (warp 1 also owns the 512 TMEM columns):
//              QK of tile t is issued before the PV of tile t-1, so a block's scores
//              for the next tile are ready while its softmax still works on the current
//              one.  A thread that polls an mbarrier stalls until its own MMAs have
//              completed, so a single issuer would serialise the blocks; two overlap.
//   warps 4-11 softmax for M-block 0 (warps 4-7) and 1 (warps 8-11), one row per thread
// The control warpgroup (warps 0-3) hands registers to the softmax warpgroups with
// setmaxnreg once the prologue is done.
// TMEM: U double-buffered per M-block, U_{b,x} at 64*(2b+x); O_b at 256 + b*d_h.  W
// overwrites the first half of U_{b,x} once the scores are read (bf16 pairs).
// Shared basis (B_K, B_V shared across tokens, same page, 优点与创新 5): the b^K, b^V
// tiles come from the layer's per-position tables, the same rows for every sequence
// (read through L2), and only a^K, a^V are per sequence; nothing else changes.
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
constexpr int kUW = 64;                     // U columns per tile (= KT * R rows of b^K)
constexpr uint32_t kBox = kUW * 128;        // one TMA box: 64 rows x 128 bytes
constexpr float kRescale = 8.f;             // lazy rescale threshold (log2 units)
// a^K, a^V tiles transposed to one row per head (R = 2, h = 16): a row holds the tile's
// 32 keys x (2 bf16) = 128 bytes, padded to 144 so that 16 heads spread over the banks
constexpr int kATS = 2;                     // transposed tiles in flight
constexpr uint32_t kATPitch = 144;

struct PrefillTcArgs {
    const __nv_bfloat16* a_q;     // [T][H][Rq]
    const __nv_bfloat16* b_q;     // [T][Rq][DH]
    const __nv_bfloat16* ca_k;    // [B][cap][H][R]
    const __nv_bfloat16* ca_v;
    __nv_bfloat16* out;           // [T][H][DH]
    int S, H, Rq, cap, n_qblocks, qpb, stages;
    int bcap;                     // B_K / B_V rows between sequences: cap, or 0 (shared basis)
    int cache_batch;              // sequences the cache holds (bounds checks)
    long long T;                  // query rows (bounds checks)
    int qstage;                   // the CTA's a^Q, b^Q block is bulk-copied into the last stage
    uint32_t qa_pad;              // ... with b^Q at this offset (after a^Q, 128-aligned)
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

// ---- packed path (R = 2, h = 16): the b^K / b^V tiles are loaded rank-major (row
// s*KT + j), so U and W hold rank 0 of the tile's 32 keys, then rank 1, and two
// consecutive keys sit in adjacent columns.  The scores of a key pair are then one pair
// of f32x2 FMAs, p converts to bf16 for both keys at once, and W is two bf16x2 products.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ void lds_v2u64(uint32_t addr, uint64_t& a, uint64_t& b) {
    asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(addr));
}

// Transposed a-factor rows of one head for the packed path: a^K as fp32 [rank][32 keys]
// (256 B, padded to 272) and a^V as bf16 [rank][32 keys] (128 B, padded to 144).
constexpr uint32_t kPkPitchK = 272, kPkPitchV = 144;

// One pass over the tile (packed path) for this thread's row (i, h) against m_ref:
// d_j = a^K_{j,0} U_{0,j} + a^K_{j,1} U_{1,j} - m_ref.  MAXONLY: out = max_j d_j.
// Otherwise p_j = 2^d_j, out = sum_j p_j, and wp = W in K order (rank, key), packed
// as bf16 pairs of consecutive keys.  MASKED applies j <= p_i (diagonal tiles).
template <bool MASKED, bool MAXONLY>
__device__ __forceinline__ void softmax_pass_pk(const uint32_t (&u)[64], uint32_t akrow, uint32_t avrow,
                                                int j0, int p_i, float m_ref, float& out,
                                                uint32_t (&wp)[32]) {
    const uint64_t mneg = f2pack(-m_ref, -m_ref);
    uint64_t acc2[2] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
    float mxa[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < 4; ++c) {                       // 8 keys per chunk
        uint64_t a0[4], a1[4];
        lds_v2u64(akrow + 32u * c, a0[0], a0[1]);
        lds_v2u64(akrow + 32u * c + 16u, a0[2], a0[3]);
        lds_v2u64(akrow + 128u + 32u * c, a1[0], a1[1]);
        lds_v2u64(akrow + 128u + 32u * c + 16u, a1[2], a1[3]);
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
        if constexpr (!MAXONLY) {
            v0 = lds_v4(avrow + 16u * c);
            v1 = lds_v4(avrow + 64u + 16u * c);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int j = 8 * c + 2 * q;
            const uint64_t u0 = f2pack(__uint_as_float(u[j]), __uint_as_float(u[j + 1]));
            const uint64_t u1 = f2pack(__uint_as_float(u[32 + j]), __uint_as_float(u[33 + j]));
            float dl, dh;
            f2unpack(fma2(a1[q], u1, fma2(a0[q], u0, mneg)), dl, dh);
            if (MASKED) {
                dl = (j0 + j <= p_i) ? dl : -INFINITY;
                dh = (j0 + j + 1 <= p_i) ? dh : -INFINITY;
            }
            if constexpr (MAXONLY) {
                mxa[q] = fmaxf(mxa[q], fmaxf(dl, dh));
            } else {
                const float pl = ex2(dl), ph = ex2(dh);
                acc2[q & 1] = add2(acc2[q & 1], f2pack(pl, ph));
                const __nv_bfloat162 pb = __floats2bfloat162_rn(pl, ph);
                const uint32_t av0 = (&v0.x)[q], av1 = (&v1.x)[q];
                const __nv_bfloat162 w0 = __hmul2(pb, *reinterpret_cast<const __nv_bfloat162*>(&av0));
                const __nv_bfloat162 w1 = __hmul2(pb, *reinterpret_cast<const __nv_bfloat162*>(&av1));
                uint32_t x0 = *reinterpret_cast<const uint32_t*>(&w0), x1 = *reinterpret_cast<const uint32_t*>(&w1);
                if (MASKED) {
                    // a key past p_i contributes exactly 0 whatever its a^V holds
                    const uint32_t keep = (pl != 0.f ? 0x0000ffffu : 0u) | (ph != 0.f ? 0xffff0000u : 0u);
                    x0 &= keep;
                    x1 &= keep;
                }
                wp[4 * c + q] = x0;
                wp[16 + 4 * c + q] = x1;
            }
        }
    }
    if constexpr (MAXONLY) {
        out = fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3]));
    } else {
        float a0l, a0h, a1l, a1h;
        f2unpack(acc2[0], a0l, a0h);
        f2unpack(acc2[1], a1l, a1h);
        out = (a0l + a0h) + (a1l + a1h);
    }
}

// One pass of the softmax over a key tile for this thread's row (i, h), relative to a
// reference max m_ref: d_j = sum_s a^K_{j,h,s} U_{(j,s)} - m_ref (log2 units), mx =
// max_j d_j, p_j = 2^d_j, lsum = sum_j p_j, and the W row (p_j a^V_{j,h,s}) in K order
// (j, s) packed as bf16 pairs.  MASKED applies the causal bound j <= p_i (diagonal tiles).
template <int R, bool MASKED, int HS_, bool AT = false>
__device__ __forceinline__ void softmax_pass(uint32_t u_addr, const __nv_bfloat16* ak,
                                             const __nv_bfloat16* av, int H, int h, int j0, int p_i,
                                             float m_ref, float& mx, float& lsum, uint32_t (&wp)[32]) {
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
        {
            constexpr int hf = 0;
            uint32_t u[64];
            tmem_ld32(u_addr, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
            tmem_ld32(u_addr + 32u, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
            uint32_t wa[32], wv[32];
            if constexpr (AT) {
                // ak, av point at this head's transposed rows: 4 keys per 16-byte load
                const uint32_t k4 = smem_u32(ak), v4 = smem_u32(av);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 x = lds_v4(k4 + 16u * c), y = lds_v4(v4 + 16u * c);
                    wa[4 * c] = x.x; wa[4 * c + 1] = x.y; wa[4 * c + 2] = x.z; wa[4 * c + 3] = x.w;
                    wv[4 * c] = y.x; wv[4 * c + 1] = y.y; wv[4 * c + 2] = y.z; wv[4 * c + 3] = y.w;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    wa[q] = lds_u32(smem_u32(akr) + 4u * q * HS);
                    wv[q] = lds_u32(smem_u32(avr) + 4u * q * HS);
                }
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
    {
        constexpr int hf = 0;
        uint32_t u[64];
        tmem_ld32(u_addr, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
        tmem_ld32(u_addr + 32u, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
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
    constexpr int KT = kUW / R;            // keys per tile
    constexpr int NB = DH / 64;            // 64-wide column blocks of d_h
    // d_h = 64: q~ lives in TMEM (columns 384.., bf16 pairs) and QK reads it from there;
    // d_h = 128 leaves no TMEM for it, so q~ stays in shared memory
    constexpr bool QT = DH == 64;
    constexpr uint32_t kQCol = 256u + 2u * DH;
    constexpr uint32_t kQBytes = QT ? 0u : NB * 256u * 128u;
    constexpr int UW = kUW;                // U columns per tile and M-block

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sq = smem;                                   // q~, [NB][256 rows][128 B]
    uint8_t* stg = smem + kQBytes;                        // stages
    // R = 2 at h = 16: warp 3 transposes each tile's a^K, a^V into kATS row-per-head buffers
    constexpr bool AT = R == 2 && HC == 16;
    // ... and its softmax runs the packed path on rank-major tiles
    constexpr bool PK = AT;
    constexpr uint32_t kATBytes = PK ? HC * (kPkPitchK + kPkPitchV) : AT ? 2u * HC * kATPitch : 0u;
    uint8_t* atr = stg + (size_t)a.stages * a.stage_bytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(atr + kATS * kATBytes);
    uint64_t* kv_full = bars;
    uint64_t* kv_empty = kv_full + a.stages;
    uint64_t* u_ready = kv_empty + a.stages;    // [2 blocks][2 buffers] scores in U
    uint64_t* w_ready = u_ready + 4;            // [2][2] W written over U
    uint64_t* o_ready = w_ready + 4;            // [2] a PV into O_b has completed
    uint64_t* o_done = o_ready + 2;             // [2] the last PV into O_b has completed
    uint64_t* fin = o_done + 2;                 // [2] each issuer's MMAs in flight at exit
    uint64_t* at_ready = fin + 2;               // [kATS] a transposed tile pair is written
    uint64_t* q_full = at_ready + kATS;         // [1] the staged query block has landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 1);
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
        // a stage is free once both M-blocks' issuers have committed their PV of it
        for (int s = 0; s < a.stages; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 2); }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&u_ready[i], 1);
            mbar_init(&w_ready[i], 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&o_ready[i], 1);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(&fin[0], 1);
        mbar_init(&fin[1], 1);
        for (int i = 0; i < kATS; ++i) mbar_init(&at_ready[i], 32);
        mbar_init(q_full, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) { prefetch_tensormap(&tmk); prefetch_tensormap(&tmv); }
    if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // K/V tile t into stage t % stages (the producer thread); false if an index check failed
    auto issue_tile = [&](int t) -> bool {
        const uint32_t full_bytes = 2u * NB * kBox;
        const int s = t % a.stages;
        const int j0 = t * KT;
        const int rows_a = min(KT, a.cap - j0);
        // the a-factor bulk copies read rows (b, j0 .. j0+rows_a) of the cache
        if (!in_bounds(b < a.cache_batch && rows_a > 0, a.err)) { *abort = 1; return false; }
        const uint32_t abytes = (uint32_t)rows_a * H * R * 2u;
        mbar_arrive_expect_tx(&kv_full[s], full_bytes + 2u * abytes);
        const int yb = b * a.bcap + j0;             // B row of key j0
        const int y = yb * R;
#pragma unroll
        for (int cb = 0; cb < NB; ++cb) {
            if constexpr (PK) {
                // rank-major box: (column, key, rank) = (cb*64, key of j0, 0)
                tma_load_3d(stage_bk(s) + cb * kBox, &tmk, &kv_full[s], cb * 64, yb, 0);
                tma_load_3d(stage_bv(s) + cb * kBox, &tmv, &kv_full[s], cb * 64, yb, 0);
            } else {
                tma_load_2d(stage_bk(s) + cb * kBox, &tmk, &kv_full[s], cb * 64, y);
                tma_load_2d(stage_bv(s) + cb * kBox, &tmv, &kv_full[s], cb * 64, y);
            }
        }
        const long long ea = ((long long)b * a.cap + j0) * H * R;
        bulk_load((void*)stage_ak(s), a.ca_k + ea, abytes, &kv_full[s]);
        bulk_load((void*)stage_av(s), a.ca_v + ea, abytes, &kv_full[s]);
        return true;
    };

    // The first K/V tiles go out before the prologue, so their latency overlaps it; with a
    // staged query block the last stage holds the CTA's a^Q, b^Q until the prologue ends.
    int t_pre = 0;
    if (warp == 0 && lane == 0) {
        if (a.qstage) {
            const long long tq = (long long)b * a.S + q0;
            const uint32_t qab = (uint32_t)nq * H * a.Rq * 2u, qbb = (uint32_t)nq * a.Rq * DH * 2u;
            uint8_t* qs = stg + (size_t)(a.stages - 1) * a.stage_bytes;
            mbar_arrive_expect_tx(q_full, qab + qbb);
            bulk_load(qs, a.a_q + tq * H * a.Rq, qab, q_full);
            bulk_load(qs + a.qa_pad, a.b_q + tq * a.Rq * DH, qbb, q_full);
        }
        const int pre = min(n_tiles, a.qstage ? a.stages - 1 : a.stages);
        for (; t_pre < pre; ++t_pre)
            if (!issue_tile(t_pre)) break;
    }

    // ---- prologue: q~ rows by the 256 softmax threads, into TMEM (QT) or into shared
    // memory (bf16, 128-byte swizzled K-major)
    if (warp >= 4) {
        const int row = threadIdx.x - 128;                // 0..255
        const int i_loc = row / H, h = row - (row / H) * H;
        const bool vq = i_loc < nq && in_bounds((long long)b * a.S + q0 + i_loc < a.T, a.err);
        const long long t = (long long)b * a.S + q0 + (vq ? i_loc : 0);
        // q~ = qscale * sum_r a^Q_r b^Q_r; TPA-KVonly (Rq = 0): qscale * q[t][h][:]
        const int nr = a.Rq > 0 ? a.Rq : 1;
        // staged: a^Q, b^Q of the CTA's queries are in shared memory (one bulk round trip
        // instead of ~Rq * d_h / 8 dependent global loads per thread)
        const uint8_t* qs = stg + (size_t)(a.stages - 1) * a.stage_bytes;
        if (a.qstage) mbar_wait(q_full, 0u, lim, a.err, abort);
        const __nv_bfloat16* aqp = a.qstage ? reinterpret_cast<const __nv_bfloat16*>(qs) + (i_loc * H + h) * a.Rq
                                            : a.a_q + (t * H + h) * a.Rq;
        // rank loops unrolled to the supported maximum (16) and predicated, so that aq
        // stays in registers (a run-time trip count put it in local memory)
        float aq[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) aq[r] = (vq && r < a.Rq) ? __bfloat162float(aqp[r]) * a.qscale : 0.f;
        if (a.Rq == 0) aq[0] = vq ? a.qscale : 0.f;
        const __nv_bfloat16* bq = a.qstage ? reinterpret_cast<const __nv_bfloat16*>(qs + a.qa_pad) + i_loc * a.Rq * DH
                                : a.Rq > 0 ? a.b_q + t * a.Rq * DH : a.b_q + (t * H + h) * DH;
        uint32_t qw[QT ? DH / 2 : 1];
#pragma unroll
        for (int k8 = 0; k8 < DH; k8 += 8) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (vq) {
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    if (r >= nr) break;
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
            if constexpr (QT) {
                qw[k8 / 2] = w.x; qw[k8 / 2 + 1] = w.y; qw[k8 / 2 + 2] = w.z; qw[k8 / 2 + 3] = w.w;
            } else {
                const int cb = k8 >> 6;
                *reinterpret_cast<uint4*>(sq + cb * (256u * 128u) + sw128_offset(row, (k8 & 63) * 2)) = w;
            }
        }
        if constexpr (QT) {
            const int bl = row >> 7;
            tmem_st32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + kQCol + (uint32_t)bl * (DH / 2), qw);
            tmem_st_wait();
        } else {
            fence_proxy_async_smem();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp < 4) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
      if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int t = t_pre;                                // tiles issued before the prologue
            for (; t < n_tiles && !*abort; ++t) {
                const int s = t % a.stages;
                if (t >= a.stages &&
                    !mbar_wait(&kv_empty[s], (uint32_t)((t / a.stages - 1) & 1), lim, a.err, abort))
                    break;
                if (!issue_tile(t)) break;
            }
            for (int s = 0; s < a.stages; ++s) {          // drain issued copies
                const int fills = t > s ? (t - s - 1) / a.stages + 1 : 0;
                if (fills > 0)
                    drain_wait(&kv_full[s], (uint32_t)((fills - 1) & 1));
            }
            if (a.qstage) drain_wait(q_full, 0u);
        }
      } else if (warp <= 2) {
        // ------------------------------------------------------------ MMA issuers
        // Warp 1 issues every MMA of M-block 0, warp 2 those of M-block 1.  An issuing
        // thread that polls an mbarrier waits there until its own MMAs in flight have
        // completed; with one issuer per block, that wait overlaps the other block's MMAs.
        if (lane == 0) {
            const int bl = warp - 1;
            const uint32_t idesc_qk = idesc_bf16(128, UW, 0, 0);
            const uint32_t idesc_pv = idesc_bf16(128, DH, 0, 1);
            const uint32_t q_base = smem_u32(sq) + (uint32_t)bl * 128u * 128u;
            const uint32_t o_col = tmem + 256u + (uint32_t)bl * DH;
            // U_{bl, t&1} = q~_bl . b^K(t)^T, b^K from stage st
            auto issue_qk = [&](int t, int st) {
                const uint32_t bk = smem_u32(stage_bk(st));
                const uint32_t u_col = tmem + (uint32_t)(2 * bl + (t & 1)) * kUW;
#pragma unroll
                for (int k = 0; k < DH / 16; ++k) {
                    const uint32_t cb = (uint32_t)(k >> 2), kk = (uint32_t)(k & 3) * 32u;
                    const uint64_t bdesc = smem_desc(bk + cb * kBox + kk, 16, 1024, kSwizzle128);
                    if constexpr (QT)
                        mma_ts(u_col, tmem + kQCol + (uint32_t)bl * (DH / 2) + (uint32_t)k * 8u, bdesc, idesc_qk,
                               k > 0 ? 1u : 0u);
                    else
                        mma_ss(u_col, smem_desc(q_base + cb * 256u * 128u + kk, 16, 1024, kSwizzle128), bdesc,
                               idesc_qk, k > 0 ? 1u : 0u);
                }
                mma_commit(&u_ready[2 * bl + (t & 1)]);
            };
            // every poll (and every shared-memory read) made by this thread waits for its
            // MMAs in flight, so the loop keeps them to the one wait it needs per tile
            bool ok = mbar_wait(&kv_full[0], 0u, lim, a.err, abort);
            if (ok) { tc_fence_after(); issue_qk(0, 0); }
            if (ok && n_tiles > 1 && (ok = mbar_wait(&kv_full[1], 0u, lim, a.err, abort))) {
                tc_fence_after();
                issue_qk(1, 1);
            }
            // Steady state: wait for the stage of tile t+2 (this also drains PV(t-1) and
            // QK(t+1), while the softmax still works on t), then for W(t), then PV(t) and
            // QK(t+2) back to back.  QK(t+2) overwrites U_{bl, t&1} after PV(t) has read
            // W from it (one issuer, in order).  s0 = stage of tile t; s2, ph2 = stage
            // and parity of tile t+2.
            int s0 = 0, s2 = 2;
            uint32_t ph2 = 0;
            for (int t = 0; ok && t < n_tiles; ++t) {
                const bool next = t + 2 < n_tiles;
                if (next && !mbar_wait(&kv_full[s2], ph2, lim, a.err, abort)) break;
                if (!mbar_wait(&w_ready[2 * bl + (t & 1)], (uint32_t)((t >> 1) & 1), lim, a.err, abort)) break;
                // block 0's softmax clears the b^V rows past the valid keys of the last
                // tile before it hands over its W; block 1's PV reads the same stage
                if (bl == 1 && t == n_tiles - 1 && t * KT + KT > kv_len &&
                    !mbar_wait(&w_ready[t & 1], (uint32_t)((t >> 1) & 1), lim, a.err, abort))
                    break;
                tc_fence_after();
                // O_bl += W_bl(t) . b^V(t)
                const uint32_t bv = smem_u32(stage_bv(s0));
                const uint32_t w_col = tmem + (uint32_t)(2 * bl + (t & 1)) * kUW;
#pragma unroll
                for (int k = 0; k < UW / 16; ++k)
                    mma_ts(o_col, w_col + (uint32_t)k * 8u, smem_desc(bv + (uint32_t)k * 2048u, kBox, 1024, kSwizzle128),
                           idesc_pv, (t > 0 || k > 0) ? 1u : 0u);
                mma_commit(&o_ready[bl]);
                if (t == n_tiles - 1) mma_commit(&o_done[bl]);
                mma_commit(&kv_empty[s0]);
                if (next) issue_qk(t + 2, s2);
                s0 = s0 + 1 == a.stages ? 0 : s0 + 1;
                if (++s2 == a.stages) { s2 = 0; ph2 ^= 1u; }
            }
            // every MMA this thread issued has completed before TMEM is released
            mma_commit(&fin[bl]);
            drain_wait(&fin[bl], 0);
        }
      } else if constexpr (AT) {
        // ------------------------------------------------------------ a-tile transpose
        // warp 3: a^K, a^V of tile t from [key][head] pairs to one row per head, into
        // buffer t % kATS once both M-blocks' softmax have finished tile t - kATS
        constexpr int kWords = KT * HC;                  // (key, head) pairs per tile
        int s = 0;
        uint32_t ph = 0;
        for (int t = 0; t < n_tiles; ++t) {
            bool good = mbar_wait(&kv_full[s], ph, lim, a.err, abort);
            if (good && t >= kATS) {
                const int tp = t - kATS;
                good = mbar_wait(&w_ready[tp & 1], (uint32_t)((tp >> 1) & 1), lim, a.err, abort) &&
                       mbar_wait(&w_ready[2 + (tp & 1)], (uint32_t)((tp >> 1) & 1), lim, a.err, abort);
            }
            if (__any_sync(0xffffffffu, !good)) break;
            const uint32_t sk = smem_u32(stage_ak(s)), sv = smem_u32(stage_av(s));
            uint8_t* dbase = atr + (t % kATS) * kATBytes;
            if constexpr (PK) {
                // a^K as fp32 [head][rank][key], a^V as bf16 [head][rank][key]
                float* dk = reinterpret_cast<float*>(dbase);
                uint16_t* dv = reinterpret_cast<uint16_t*>(dbase + HC * kPkPitchK);
#pragma unroll 4
                for (int w = lane; w < kWords; w += 32) {
                    const int j = w / HC, hh = w % HC;
                    const uint32_t kw = lds_u32(sk + 4u * w), vw = lds_u32(sv + 4u * w);
                    dk[hh * (kPkPitchK / 4) + j] = bf16lo(kw);
                    dk[hh * (kPkPitchK / 4) + 32 + j] = bf16hi(kw);
                    dv[hh * (kPkPitchV / 2) + j] = (uint16_t)(vw & 0xffffu);
                    dv[hh * (kPkPitchV / 2) + 32 + j] = (uint16_t)(vw >> 16);
                }
            } else {
                uint32_t* dk = reinterpret_cast<uint32_t*>(dbase);
                uint32_t* dv = dk + HC * (kATPitch / 4);
#pragma unroll 4
                for (int w = lane; w < kWords; w += 32) {
                    const int j = w / HC, hh = w % HC;
                    dk[hh * (kATPitch / 4) + j] = lds_u32(sk + 4u * w);
                    dv[hh * (kATPitch / 4) + j] = lds_u32(sv + 4u * w);
                }
            }
            mbar_arrive(&at_ready[t % kATS]);
            if (++s == a.stages) { s = 0; ph ^= 1u; }
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
        const uint32_t o_col = 256u + (uint32_t)bl * DH;
        float m_use = -INFINITY, l = 0.f;
        bool alive = true;
        for (int t = 0; t < n_tiles; ++t) {
            const int ub = 2 * bl + (t & 1);
            // leave together: the warp votes below need every lane
            bool got = mbar_wait(&u_ready[ub], (uint32_t)((t >> 1) & 1), lim, a.err, abort);
            if constexpr (AT) got = got && mbar_wait(&at_ready[t % kATS], (uint32_t)((t / kATS) & 1), lim, a.err, abort);
            if (__any_sync(0xffffffffu, !got)) { alive = false; break; }
            tc_fence_after();
            const uint32_t u_addr = lane_addr + (uint32_t)ub * kUW;
            const int s = t % a.stages;
            const int j0 = t * KT;
            const __nv_bfloat16* ak;
            const __nv_bfloat16* av;
            if constexpr (AT) {
                ak = reinterpret_cast<const __nv_bfloat16*>(atr + (t % kATS) * kATBytes + h * kATPitch);
                av = reinterpret_cast<const __nv_bfloat16*>(atr + (t % kATS) * kATBytes + (HC + h) * kATPitch);
            } else {
                ak = stage_ak(s);
                av = stage_av(s);
            }
            const bool masked = j0 + KT - 1 > p0;        // same for every row of the CTA
            uint32_t wp[32];
            float mx = -INFINITY, lsum = 0.f;
            bool ok = false;
            if constexpr (PK) {
                uint32_t u[64];
                tmem_ld32(u_addr, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
                tmem_ld32(u_addr + 32u, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
                const uint32_t akrow = smem_u32(atr + (t % kATS) * kATBytes) + (uint32_t)h * kPkPitchK;
                const uint32_t avrow = smem_u32(atr + (t % kATS) * kATBytes + HC * kPkPitchK) + (uint32_t)h * kPkPitchV;
                tmem_ld_wait();
                if (t > 0) {
                    // one pass against the running max; if the tile's sum stays within
                    // 2^8, so does every term, and no rescale is needed
                    if (masked) softmax_pass_pk<true, false>(u, akrow, avrow, j0, p_i, m_use, lsum, wp);
                    else softmax_pass_pk<false, false>(u, akrow, avrow, j0, p_i, m_use, lsum, wp);
                    ok = lsum <= 256.f;
                }
                if (__all_sync(0xffffffffu, ok)) {
                    l += lsum;
                } else {
                    // first tile, or a score well above the running max: exact max, rescale O
                    const float m_ref = t == 0 ? 0.f : m_use;
                    if (masked) softmax_pass_pk<true, true>(u, akrow, avrow, j0, p_i, m_ref, mx, wp);
                    else softmax_pass_pk<false, true>(u, akrow, avrow, j0, p_i, m_ref, mx, wp);
                    const float m_new = t == 0 ? mx : m_use + fmaxf(mx, 0.f);
                    const float alpha = t == 0 ? 1.f : ex2(m_use - m_new);
                    if (t > 0) l *= alpha;
                    if (t > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                        // O row *= alpha, once PV(t-1) into O has completed
                        const bool pv_done = mbar_wait(&o_ready[bl], (uint32_t)((t - 1) & 1), lim, a.err, abort);
                        if (__any_sync(0xffffffffu, !pv_done)) { alive = false; break; }
                        tc_fence_after();
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
                    if (masked) softmax_pass_pk<true, false>(u, akrow, avrow, j0, p_i, m_use, lsum, wp);
                    else softmax_pass_pk<false, false>(u, akrow, avrow, j0, p_i, m_use, lsum, wp);
                    l += lsum;
                }
            } else {
            if (t > 0) {
                // common case: one pass against the running max
                if (masked) softmax_pass<R, true, HC, AT>(u_addr, ak, av, H, h, j0, p_i, m_use, mx, lsum, wp);
                else softmax_pass<R, false, HC, AT>(u_addr, ak, av, H, h, j0, p_i, m_use, mx, lsum, wp);
                ok = mx <= kRescale;
            }
            if (__all_sync(0xffffffffu, ok)) {
                l += lsum;
            } else {
                // first tile, or the max rose by more than 2^kRescale: exact max, rescale O
                if (t == 0) {
                    if (masked) softmax_pass<R, true, HC, AT>(u_addr, ak, av, H, h, j0, p_i, 0.f, mx, lsum, wp);
                    else softmax_pass<R, false, HC, AT>(u_addr, ak, av, H, h, j0, p_i, 0.f, mx, lsum, wp);
                }
                const float m_new = (t == 0) ? mx : (mx > kRescale ? m_use + mx : m_use);
                const float alpha = (t == 0) ? 1.f : ex2(m_use - m_new);
                if (t > 0) l *= alpha;
                if (t > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                    // O row *= alpha, once PV(t-1) into O has completed
                    const bool pv_done = mbar_wait(&o_ready[bl], (uint32_t)((t - 1) & 1), lim, a.err, abort);
                    if (__any_sync(0xffffffffu, !pv_done)) { alive = false; break; }
                    tc_fence_after();
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
                if (masked) softmax_pass<R, true, HC, AT>(u_addr, ak, av, H, h, j0, p_i, m_use, mx, lsum, wp);
                else softmax_pass<R, false, HC, AT>(u_addr, ak, av, H, h, j0, p_i, m_use, mx, lsum, wp);
                l += lsum;
            }
            }
            // W over the first half of U (the scores have all been read)
            tmem_st32(u_addr, wp);
            tmem_st_wait();
            if (bl == 0 && t == n_tiles - 1 && j0 + KT > kv_len) {
                // keys at or past the valid length: clear their b^V rows so that
                // 0 * (whatever the cache holds there) stays 0 in the PV product
                // (tile rows are (key, rank), or rank-major s*KT + key on the packed path)
                uint8_t* bv = stage_bv(s);
                const int nv = kv_len - j0;                 // valid keys in the tile
                for (int idx = threadIdx.x - 128; idx < UW; idx += 128) {
                    const int key = PK ? idx % KT : idx / R;
                    if (key < nv) continue;
                    for (int cb = 0; cb < NB; ++cb) {
                        uint4* pz = reinterpret_cast<uint4*>(bv + cb * kBox + idx * 128);
#pragma unroll
                        for (int e = 0; e < 8; ++e) pz[e] = make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            mbar_arrive(&w_ready[ub]);
        }
        const bool done_ok = alive && mbar_wait(&o_done[bl], 0u, lim, a.err, abort);
        if (__all_sync(0xffffffffu, done_ok)) {
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
    constexpr int KT = kUW / R;
    constexpr int NB = DH / 64;
    a.a_bytes = (uint32_t)(KT * a.H * R * 2);
    const uint32_t a_pad = (a.a_bytes + 127u) & ~127u;
    a.stage_bytes = ((2u * NB * kBox + 2u * a_pad) + 1023u) & ~1023u;
    const uint32_t q_bytes = DH == 64 ? 0u : NB * 256u * 128u;   // q~ in TMEM at d_h 64
    const uint32_t at_bytes = (R == 2 && HC == 16) ? kATS * HC * (kPkPitchK + kPkPitchV) : 0u;
    const uint32_t budget = 227u * 1024u - 1024u - 512u - q_bytes - at_bytes;
    a.stages = std::min(8, (int)(budget / a.stage_bytes));
    if (a.stages < 3) return cudaErrorInvalidValue;   // QK(t+2) and PV(t) use different stages
    CUtensorMap tmk, tmv;
    // B rows: every sequence's (contextual), or one per-position table (shared basis)
    const uint64_t b_keys = (uint64_t)(a.bcap ? c.batch : 1) * (uint64_t)c.capacity;
    if constexpr (R == 2 && HC == 16) {
        // packed path: [d_h][key][rank] with rank outermost, so a box of KT keys x 2
        // ranks lands rank-major (row s*KT + key)
        const uint64_t dims[3] = {(uint64_t)DH, b_keys, (uint64_t)R};
        const uint64_t stride[2] = {(uint64_t)R * DH * 2, (uint64_t)DH * 2};
        const uint32_t box[3] = {64, (uint32_t)KT, (uint32_t)R};
        if (!make_tmap_bf16(&tmk, c.b_k, 3, dims, stride, box) || !make_tmap_bf16(&tmv, c.b_v, 3, dims, stride, box))
            return cudaErrorInvalidValue;
    } else {
        const uint64_t dims[2] = {(uint64_t)DH, b_keys * R};
        const uint64_t stride[1] = {(uint64_t)DH * 2};
        const uint32_t box[2] = {64, (uint32_t)kUW};
        if (!make_tmap_bf16(&tmk, c.b_k, 2, dims, stride, box) || !make_tmap_bf16(&tmv, c.b_v, 2, dims, stride, box))
            return cudaErrorInvalidValue;
    }
    // the query block (a^Q then b^Q of qpb queries) can borrow the last stage at the start
    a.qa_pad = ((uint32_t)a.qpb * a.H * a.Rq * 2u + 127u) & ~127u;
    a.qstage = (a.Rq > 0 && (a.H * a.Rq) % 8 == 0 &&
                a.qa_pad + (uint32_t)a.qpb * a.Rq * DH * 2u <= a.stage_bytes) ? 1 : 0;
    const size_t smem = 1024 + q_bytes + (size_t)a.stages * a.stage_bytes + at_bytes + (2 * a.stages + 15 + kATS) * 8 + 16;
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
    if (s.Rq < 0 || s.Rq > 16) return false;          // 0: TPA-KVonly, the query is given
    // at least three stages of (b^K, b^V boxes + a^K, a^V tiles of 128*h bytes) beside q~
    const uint32_t nb = (uint32_t)s.Dh / 64u;
    const uint32_t a_pad = (128u * (uint32_t)s.H + 127u) & ~127u;
    const uint32_t stage = ((2u * nb * kBox + 2u * a_pad) + 1023u) & ~1023u;
    const uint32_t at_bytes = (s.Rk == 2 && s.H == 16) ? kATS * 16u * (kPkPitchK + kPkPitchV) : 0u;
    return 227u * 1024u - 1024u - 512u - nb * 256u * 128u - at_bytes >= 3u * stage;
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
    a.bcap = (int)b_seq_rows(s, c);
    a.cache_batch = c.batch;
    a.T = (long long)batch * seqlen;
    a.qpb = 256 / s.H;
    a.n_qblocks = (seqlen + a.qpb - 1) / a.qpb;
    a.qscale = 1.4426950408889634f / ((float)(s.Rq > 0 ? s.Rq : 1) * (float)s.Rk * std::sqrt((float)s.Dh));
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
