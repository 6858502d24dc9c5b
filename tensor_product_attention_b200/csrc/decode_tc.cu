// Decode from the factor cache on tcgen05 tensor cores (bf16, fp32 accumulate).
//
// One query per sequence at position len-1 attends to the cached keys 0..len-1
// ("【拜读】Tensor Product Attention Is All You Need…" (coreui.cn), 代码 前向传播: the
// cache is written, then read over [:start_pos+seqlen]), reading only the factors; B_K
// is used as cached, already rotated (same page, 关键问题及回答 问题2).  With the query
// folded once per sequence, q~_h = log2(e)/(R_Q R_K sqrt(d_h)) sum_r a^Q_{h,r} b^Q_r
// (or the given per-head q for TPA-KVonly), a tile of KT = 128/R keys costs:
//   U^T  = b^K . q~^T     tcgen05, M = 128 rows (key j, rank s), N = h, K = d_h
//   score_h(j) = sum_s a^K_{j,h,s} U^T_{(j,s),h}      one thread per row, shfl over s
//   W^T_{(j,s),h} = 2^(score - m_h) a^V_{j,h,s}        bf16, to shared memory
//   O^T += b^V^T . W^T    tcgen05, M = d_h (A = b^V tile read MN-major), N = h, K = 128
// HBM-bound: only (R_K + R_V)(h + d_h) factor elements per key are read.  Staging all
// of them through shared memory runs at ~20 B per cycle per SM, the rate of the
// measured HBM copy.
//
// Scheduling: a persistent grid of one CTA per SM walks the key tiles of all
// sequences concatenated; CTA c takes tiles [c*N/G, (c+1)*N/G), so ragged lengths are
// balanced exactly.  Each (CTA, sequence) overlap ("part") writes its partial softmax
// state (m_h, l_h, O^T) to the workspace; the combine kernel merges the parts of a
// sequence in a fixed order.  The softmax keeps a CTA-wide reference max per head and
// only revisits it (rescaling O^T in tensor memory) when a score exceeds it by more
// than 2^8, so a tile normally needs one pass and one barrier.
//
// Warp roles: warp 0 TMA for the K ring (b^K tiles, 128-byte swizzle, and a^K/a^V),
// warp 2 TMA for the V ring (b^V tiles), warp 1 TMEM owner and QK issuer, warp 3 PV
// issuer, warps 4.. softmax (4 warps per 16 heads; TMEM lane = row).  At h 32 (two
// head groups) warp 1 issues both QK and PV and the softmax starts at warp 3: the
// 352-thread CTA keeps a register cap of 186 (a fourth control warp measured 4% slower
// there, while at h 16 the separate PV issuer gains 5%).  TMEM: U^T double-buffered
// (2 x h columns) and O^T (h).
//
// Shared basis (B_K, B_V shared across tokens, same page, 优点与创新 5), kernel SB: b^K
// tiles come from the layer's per-position table (row j = the key basis rotated at j,
// the same for every sequence, so it is read through L2).  Every value row of rank s is
// the basis b^V_s, so O_h = sum_s (sum_j p_{j,h} a^V_{j,h,s}) b^V_s: the softmax threads
// keep sum_j p a^V in registers (each row has one rank) and apply the basis once per
// part; there is no PV MMA, no V ring and no W^T.  Per key only the (R_K + R_V) h A
// factors come from the sequence's cache.  At h 16 (PAIR) two sequences share each
// key tile: the stage holds one table tile and both sequences' A tiles, QK has 32
// columns (q~ of sequence 2u in rows 0..15, of 2u+1 in rows 16..31), head group g
// serves member g, and the plan walks units of two sequences (c_first per unit, each
// member with its own consecutive parts).  A member with no valid key in a whole part
// leaves m = -inf, l = 0, O = 0, which the merge weighs as zero.
#include <algorithm>
#include <cmath>

#include "tpa_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace tpa {

namespace {
using namespace sm100;

constexpr uint32_t kBox = 128 * 128;     // one TMA box: 128 rows x 128 bytes
constexpr float kTau = 8.f;              // lazy rescale threshold (log2 units)
constexpr int kVS = 2;                   // V ring depth (b^V tiles, read by PV)

struct DecodeTcArgs {
    const __nv_bfloat16* q_a;      // [B][H][Rq] or null
    const __nv_bfloat16* q_b;      // [B][Rq][DH] or q [B][H][DH]
    const __nv_bfloat16* ca_k;     // [B][cap][H][R]
    const __nv_bfloat16* ca_v;
    const __nv_bfloat16* cb_v;     // shared basis: the value table (row 0 = the basis)
    float* ws_ml;                  // [parts][H][2]
    float* ws_o;                   // [parts][H][DH]
    int Rq, cap;
    int bcap;                      // B rows between sequences: cap, or 0 (shared basis)
    int asw;                       // a^K, a^V tiles by TMA with the 128-byte swizzle
    float qscale;
    uint32_t a_bytes, kstage_bytes;  // a^K (or a^V) tile; one K-ring stage (b^K, a^K, a^V)
    int ks;                          // K ring depth (2..4, as shared memory allows)
    int cache_batch;                 // sequences the cache holds (bounds checks)
    int* err;
    uint32_t wait_limit;
};

// tile bookkeeping shared by every role: which sequence / local tile a CTA tile is
template <int KT>
struct TileWalk {
    int b;           // current sequence
    __device__ void init(const DecodePlan& P, int g) {
        b = 0;
        while (P.tile_prefix[b + 1] <= g) ++b;
    }
    __device__ void advance(const DecodePlan& P, int g) {
        while (P.tile_prefix[b + 1] <= g) ++b;
    }
};

template <int DH, int HH, int R, bool SB, bool PAIR>
__global__ void __launch_bounds__(((HH == 32 && !SB) ? 96 : 128) + 32 * 4 * (HH / 16), 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                 const __grid_constant__ CUtensorMap tmak, const __grid_constant__ CUtensorMap tmav,
                 const DecodeTcArgs a, const DecodePlan P) {
    constexpr int KT = 128 / R;                 // keys per tile
    constexpr int NB = DH / 64;                 // 64-wide column blocks of d_h (1 or 2)
    constexpr int NG = HH / 16;                 // head groups of 16 (4 warps each)
    constexpr int NSM = 128 * NG;               // softmax threads
    constexpr uint32_t kQW = HH * 256u;         // q~ or W^T buffer: 2 x [HH rows][128 B]
    // PAIR (shared basis, h 16): the HH = 32 columns are two sequences' 16 heads; a tile
    // walks one unit (2u, 2u+1); head group hg serves member hg.
    static_assert(!PAIR || (SB && HH == 32), "pairs: shared-basis kernel, two sequences of 16 heads");
    constexpr int HS = PAIR ? HH / 2 : HH;      // heads per sequence
    constexpr int NM = PAIR ? 2 : 1;            // sequences per tile
    constexpr bool ONE = HH == 32 && !SB;       // h 32 contextual: one issuer warp
    constexpr int kSoft0 = ONE ? 3 : 4;         // first softmax warp

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    // Two rings: K (b^K, a^K, a^V: read by QK and the softmax) a.ks deep, and V (b^V:
    // read by PV) kVS deep, so the key side prefetches further than the value side.
    // The shared-basis kernel (SB) has no V ring and no W^T buffers.
    uint8_t* kring = smem;
    uint8_t* vring = kring + (size_t)a.ks * a.kstage_bytes;
    uint8_t* qbuf = vring + (SB ? (size_t)0 : (size_t)kVS * 2 * kBox);   // 2 x q~
    uint8_t* wbuf = qbuf + 2 * kQW;                                     // 2 x W^T
    float* red = reinterpret_cast<float*>(wbuf + (SB ? 0u : 2 * kQW));  // [NG][192] scratch
    uint64_t* bars = reinterpret_cast<uint64_t*>(red + NG * 192);
    uint64_t* k_full = bars;                     // [ks]
    uint64_t* k_empty = k_full + a.ks;           // [ks] every softmax thread is done with it
    uint64_t* v_full = k_empty + a.ks;           // [kVS]
    uint64_t* v_empty = v_full + kVS;            // [kVS] its PV has completed
    uint64_t* u_full = v_empty + kVS;            // [2]
    uint64_t* w_full = u_full + 2;               // [2]
    uint64_t* w_empty = w_full + 2;              // [2]
    uint64_t* q_ready = w_empty + 2;             // [2]
    uint64_t* o_done = q_ready + 2;              // [1]
    uint64_t* o_free = o_done + 1;               // [1]
    uint64_t* fin = o_free + 1;                  // MMAs in flight at exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    auto st_bk = [&](int s) { return kring + (size_t)s * a.kstage_bytes; };
    const uint32_t a_pad = (a.a_bytes + 127u) & ~127u;
    // member m's a^K, a^V tiles follow the b^K box
    auto st_ak = [&](int s, int m = 0) {
        return kring + (size_t)s * a.kstage_bytes + NB * kBox + (size_t)(2 * m) * a_pad;
    };
    auto st_av = [&](int s, int m = 0) {
        return kring + (size_t)s * a.kstage_bytes + NB * kBox + (size_t)(2 * m + 1) * a_pad;
    };
    auto st_bv = [&](int s) { return vring + (size_t)s * 2 * kBox; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const long long N = P.total_tiles, G = gridDim.x;
    const int g0 = (int)(c * N / G), g1 = (int)((c + 1) * N / G);
    const int n = g1 - g0;
    const uint32_t lim = a.wait_limit;

    if (threadIdx.x == 0) {
        // SB: two K-side producers (table tiles, a tiles) arrive on each stage
        for (int s = 0; s < a.ks; ++s) { mbar_init(&k_full[s], SB ? 2 : 1); mbar_init(&k_empty[s], NSM); }
        for (int s = 0; s < kVS; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&u_full[i], 1);
            mbar_init(&w_full[i], NSM);
            mbar_init(&w_empty[i], 1);
            mbar_init(&q_ready[i], 1);
        }
        mbar_init(o_done, 1);
        mbar_init(o_free, NSM);
        mbar_init(fin, (SB || ONE) ? 1 : 2);     // one commit from each MMA issuer
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmk); prefetch_tensormap(&tmv);
        prefetch_tensormap(&tmak); prefetch_tensormap(&tmav);
    }
    if (warp == 1) { tmem_alloc(tmem_slot, 128); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 2) {
        // ---------------------------------------------------------------- producers
        // warp 0: the K ring (b^K, a^K, a^V); warp 2: the V ring (b^V).  SB has no V ring:
        // there warp 0 stages the table tiles of the K ring and warp 2 its a^K, a^V tiles,
        // since the copies one thread issues complete one after another (~0.4K cycles
        // each from L2) and a stage holds up to six of them.
        const bool kside = warp == 0 || SB;
        const bool do_b = !SB || warp == 0;     // K side: the b^K (table) boxes
        const bool do_a = !SB || warp == 2;     // K side: the a^K, a^V tiles
        const int depth = kside ? a.ks : kVS;
        uint64_t* full = kside ? k_full : v_full;
        uint64_t* empty = kside ? k_empty : v_empty;
        if (lane == 0 && n > 0) {
            TileWalk<KT> tw;
            tw.init(P, g0);
            int i = 0;
            int s = 0;                 // ring slot i % depth
            uint32_t ph = 0;           // (i / depth) & 1
            for (; i < n && !*abort; ++i) {
                const int g = g0 + i;
                tw.advance(P, g);
                const int b = tw.b;
                const int j0 = (g - P.tile_prefix[b]) * KT;
                if (i >= depth && !mbar_wait(&empty[s], ph ^ 1u, lim, a.err, abort))
                    break;
                const int y = (int)(((long long)b * a.bcap + j0) * R);
                if (kside && !in_bounds(NM * b < a.cache_batch && j0 < a.cap, a.err)) { *abort = 1; break; }
                if (kside) {
                    // a^K, a^V: one TMA box each, 128-byte rows (one key at h 32, two at
                    // h 16) with the 128-byte swizzle; keys past the tensor read as zeros,
                    // so the box lands whole.  Otherwise (h 16) bulk copies of the valid rows.
                    // PAIR: both members' tiles (an odd batch's last unit loads member 0
                    // twice; its second group masks every key).
                    const int rows_a = a.asw ? KT : min(KT, a.cap - j0);
                    const uint32_t abytes = (uint32_t)rows_a * HS * R * 2u;
                    mbar_arrive_expect_tx(&full[s], (do_b ? NB * kBox : 0u) + (do_a ? 2u * NM * abytes : 0u));
                    if (do_b) {
                        tma_load_2d(st_bk(s), &tmk, &full[s], 0, y);
                        if (NB == 2) tma_load_2d(st_bk(s) + kBox, &tmk, &full[s], 64, y);
                    }
#pragma unroll
                    for (int m = 0; m < NM && do_a; ++m) {
                        const int sq = (NM * b + m < a.cache_batch) ? NM * b + m : NM * b;
                        if (a.asw) {
                            const int ya = (sq * a.cap + j0) / (128 / (HS * R * 2));
                            tma_load_2d(st_ak(s, m), &tmak, &full[s], 0, ya);
                            tma_load_2d(st_av(s, m), &tmav, &full[s], 0, ya);
                        } else {
                            const long long ea = ((long long)sq * a.cap + j0) * HS * R;
                            bulk_load(st_ak(s, m), a.ca_k + ea, abytes, &full[s]);
                            bulk_load(st_av(s, m), a.ca_v + ea, abytes, &full[s]);
                        }
                    }
                } else {
                    // the value MMA has M = 128 rows of d_h: for d_h = 64 the one box is
                    // loaded twice and output rows 64..127 (a copy of 0..63) are dropped
                    mbar_arrive_expect_tx(&full[s], 2u * kBox);
                    tma_load_2d(st_bv(s), &tmv, &full[s], 0, y);
                    tma_load_2d(st_bv(s) + kBox, &tmv, &full[s], NB == 2 ? 64 : 0, y);
                }
                if (++s == depth) { s = 0; ph ^= 1u; }
            }
            for (int s = 0; s < depth; ++s) {                   // drain issued copies
                const int fills = i > s ? (i - s - 1) / depth + 1 : 0;
                if (fills > 0)
                    drain_wait(&full[s], (uint32_t)((fills - 1) & 1));
            }
        }
    } else if (warp == 1 || (warp == 3 && !SB && !ONE)) {
        // ---------------------------------------------------------------- MMA issuers
        // h 16: warp 1 issues QK of every tile, warp 3 PV of every tile.  A thread that
        // polls an mbarrier stalls until its own MMAs have completed, so one issuer for
        // both serialised them (QK(t+1), drain, PV(t), drain); two let the waits of one
        // overlap the MMAs of the other.  h 32 (ONE): warp 1 issues both, which keeps
        // the CTA at three control warps.  Shared basis: warp 1 issues QK only.
        if (lane == 0 && n > 0) {
            if constexpr (ONE) {
            // one issuer for both streams: QK(i), then PV(i-1); at a sequence boundary the
            // previous part's last PV goes first (the softmax reads that part's O^T
            // before it builds the next q~)
            const uint32_t idesc_qk = idesc_bf16(128, HH, 0, 0);
            const uint32_t idesc_pv = idesc_bf16(128, HH, 1, 0);
            const uint32_t q0 = smem_u32(qbuf), w0 = smem_u32(wbuf);
            TileWalk<KT> twq, twp;
            twq.init(P, g0);
            twp.init(P, g0);
            int segq = -1, segp = -1;
            int prev_bq = -1, prev_bp = -1;
            int ks = 0;                // K ring slot of tile i: i % a.ks
            uint32_t kph = 0;          // (i / a.ks) & 1
            auto issue_pv = [&](int j) -> bool {
                const int g = g0 + j;
                twp.advance(P, g);
                const bool first = twp.b != prev_bp;
                if (first) { ++segp; prev_bp = twp.b; }
                const bool last = (j == n - 1) || (P.tile_prefix[twp.b + 1] <= g + 1);
                if (!mbar_wait(&w_full[j & 1], (uint32_t)((j >> 1) & 1), lim, a.err, abort)) return false;
                if (first && segp > 0 &&
                    !mbar_wait(o_free, (uint32_t)((segp - 1) & 1), lim, a.err, abort))
                    return false;
                const int s = j % kVS;
                if (!mbar_wait(&v_full[s], (uint32_t)((j / kVS) & 1), lim, a.err, abort)) return false;
                tc_fence_after();
                const uint32_t bv = smem_u32(st_bv(s));
                const uint32_t wb = w0 + (uint32_t)(j & 1) * kQW;
#pragma unroll
                for (int k = 0; k < 128 / 16; ++k) {
                    mma_ss(tmem + 2u * HH, smem_desc(bv + (uint32_t)k * 2048u, kBox, 1024, kSwizzle128),
                           smem_desc(wb + (uint32_t)(k >> 2) * (HH * 128u) + (uint32_t)(k & 3) * 32u,
                                     16, 1024, kSwizzle128),
                           idesc_pv, (first && k == 0) ? 0u : 1u);
                }
                mma_commit(&w_empty[j & 1]);
                mma_commit(&v_empty[s]);
                if (last) mma_commit(o_done);
                return true;
            };
            for (int i = 0; i <= n && !*abort; ++i) {
                bool newseg = false;
                if (i < n) {
                    twq.advance(P, g0 + i);
                    newseg = twq.b != prev_bq;
                }
                const bool pv_first = i >= 1 && (i == n || newseg);
                if (pv_first && !issue_pv(i - 1)) break;
                if (i < n) {
                    if (newseg) {
                        ++segq;
                        prev_bq = twq.b;
                        if (!mbar_wait(&q_ready[segq & 1], (uint32_t)((segq >> 1) & 1), lim, a.err, abort)) break;
                    }
                    if (!mbar_wait(&k_full[ks], kph, lim, a.err, abort)) break;
                    tc_fence_after();
                    const uint32_t bk = smem_u32(st_bk(ks));
                    const uint32_t qb = q0 + (uint32_t)(segq & 1) * kQW;
#pragma unroll
                    for (int k = 0; k < DH / 16; ++k) {
                        const uint32_t cb = (uint32_t)(k >> 2), kk = (uint32_t)(k & 3) * 32u;
                        mma_ss(tmem + (uint32_t)(i & 1) * HH,
                               smem_desc(bk + cb * kBox + kk, 16, 1024, kSwizzle128),
                               smem_desc(qb + cb * (HH * 128u) + kk, 16, 1024, kSwizzle128), idesc_qk,
                               k > 0 ? 1u : 0u);
                    }
                    mma_commit(&u_full[i & 1]);
                    if (++ks == a.ks) { ks = 0; kph ^= 1u; }
                }
                if (i >= 1 && !pv_first && !issue_pv(i - 1)) break;
            }
            } else
            if (warp == 1) {
                const uint32_t idesc_qk = idesc_bf16(128, HH, 0, 0);
                const uint32_t q0 = smem_u32(qbuf);
                TileWalk<KT> twq;
                twq.init(P, g0);
                int segq = -1, prev_bq = -1;
                int ks = 0;            // K ring slot of tile i: i % a.ks
                uint32_t kph = 0;      // (i / a.ks) & 1
                for (int i = 0; i < n && !*abort; ++i) {
                    twq.advance(P, g0 + i);
                    if (twq.b != prev_bq) {
                        ++segq;
                        prev_bq = twq.b;
                        if (!mbar_wait(&q_ready[segq & 1], (uint32_t)((segq >> 1) & 1), lim, a.err, abort)) break;
                    }
                    // U buffer i&1 is free once the softmax of tile i-2 has read it
                    if (i >= 2 && !mbar_wait(&w_full[i & 1], (uint32_t)(((i >> 1) - 1) & 1), lim, a.err, abort))
                        break;
                    if (!mbar_wait(&k_full[ks], kph, lim, a.err, abort)) break;
                    tc_fence_after();
                    const uint32_t bk = smem_u32(st_bk(ks));
                    const uint32_t qb = q0 + (uint32_t)(segq & 1) * kQW;
#pragma unroll
                    for (int k = 0; k < DH / 16; ++k) {
                        const uint32_t cb = (uint32_t)(k >> 2), kk = (uint32_t)(k & 3) * 32u;
                        mma_ss(tmem + (uint32_t)(i & 1) * HH,
                               smem_desc(bk + cb * kBox + kk, 16, 1024, kSwizzle128),
                               smem_desc(qb + cb * (HH * 128u) + kk, 16, 1024, kSwizzle128), idesc_qk,
                               k > 0 ? 1u : 0u);
                    }
                    mma_commit(&u_full[i & 1]);
                    if (++ks == a.ks) { ks = 0; kph ^= 1u; }
                }
            } else {
                const uint32_t idesc_pv = idesc_bf16(128, HH, 1, 0);
                const uint32_t w0 = smem_u32(wbuf);
                TileWalk<KT> twp;
                twp.init(P, g0);
                int segp = -1, prev_bp = -1;
                for (int j = 0; j < n && !*abort; ++j) {
                    const int g = g0 + j;
                    twp.advance(P, g);
                    const bool first = twp.b != prev_bp;
                    if (first) { ++segp; prev_bp = twp.b; }
                    const bool last = (j == n - 1) || (P.tile_prefix[twp.b + 1] <= g + 1);
                    if (!mbar_wait(&w_full[j & 1], (uint32_t)((j >> 1) & 1), lim, a.err, abort)) break;
                    if (first && segp > 0 &&
                        !mbar_wait(o_free, (uint32_t)((segp - 1) & 1), lim, a.err, abort))
                        break;
                    const int s = j % kVS;
                    if (!mbar_wait(&v_full[s], (uint32_t)((j / kVS) & 1), lim, a.err, abort)) break;
                    tc_fence_after();
                    const uint32_t bv = smem_u32(st_bv(s));
                    const uint32_t wb = w0 + (uint32_t)(j & 1) * kQW;
#pragma unroll
                    for (int k = 0; k < 128 / 16; ++k) {
                        mma_ss(tmem + 2u * HH, smem_desc(bv + (uint32_t)k * 2048u, kBox, 1024, kSwizzle128),
                               smem_desc(wb + (uint32_t)(k >> 2) * (HH * 128u) + (uint32_t)(k & 3) * 32u,
                                         16, 1024, kSwizzle128),
                               idesc_pv, (first && k == 0) ? 0u : 1u);
                    }
                    mma_commit(&w_empty[j & 1]);
                    mma_commit(&v_empty[s]);
                    if (last) mma_commit(o_done);
                }
            }
            // every MMA either issuer issued has completed before TMEM is released
            mma_commit(fin);
            drain_wait(fin, 0);
        }
    } else if (warp >= kSoft0) {
        // ---------------------------------------------------------------- softmax
        const int sw = warp - kSoft0;            // 0 .. 4*NG-1
        const int hg = sw >> 2;                  // head group (16 heads)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;       // TMEM lane = tile row (key j, rank s)
        const int jl = r / R, sr = r % R;
        const int stid = threadIdx.x - 32 * kSoft0;  // 0 .. NSM-1
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
        const int hbase = hg * 16;
        float m[16], lp[16];
        float acc[16];                           // SB: sum over keys of p a^V (this row's rank)
        TileWalk<KT> tw;
        if (n > 0) tw.init(P, g0);
        int seg = -1, prev_b = -1;
        int ks = 0;                              // K ring slot of tile i: i % a.ks
        uint32_t kph = 0;                        // (i / a.ks) & 1
        // A failed (timed-out) wait only sets `bad`; the loop is left at the end of the
        // tile by all softmax threads together (barrier 4), so that no thread is left
        // waiting at a named barrier or a warp vote that the others have skipped.
        bool bad = false;
        for (int i = 0; i < n; ++i) {
            const int g = g0 + i;
            tw.advance(P, g);
            const int b = tw.b;
            const bool first = b != prev_b;
            if (first) {
                ++seg;
                prev_b = b;
                // q~ for this sequence into buffer seg&1 (K-major, 128-byte swizzle)
                uint8_t* qb = qbuf + (size_t)(seg & 1) * kQW;
                for (int e = stid; e < HH * (DH / 8); e += NSM) {
                    const int h = e / (DH / 8), k8 = (e % (DH / 8)) * 8;
                    // column h is head qh of sequence qs (PAIR: member h / HS of the unit)
                    const int qs = NM * b + h / HS, qh = h % HS;
                    float acc[8];
#pragma unroll
                    for (int x = 0; x < 8; ++x) acc[x] = 0.f;
                    if (qs >= P.batch) {
                        // an odd batch's last unit: no second sequence (its group masks all keys)
                    } else if (a.Rq > 0) {
                        for (int rq = 0; rq < a.Rq; ++rq) {
                            const float aqv = __bfloat162float(a.q_a[((long long)qs * HS + qh) * a.Rq + rq]);
                            const uint4 raw = *reinterpret_cast<const uint4*>(a.q_b + ((long long)qs * a.Rq + rq) * DH + k8);
                            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                            for (int x = 0; x < 4; ++x) {
                                const float2 f = __bfloat1622float2(p2[x]);
                                acc[2 * x] = fmaf(aqv, f.x, acc[2 * x]);
                                acc[2 * x + 1] = fmaf(aqv, f.y, acc[2 * x + 1]);
                            }
                        }
                    } else {
                        const uint4 raw = *reinterpret_cast<const uint4*>(a.q_b + ((long long)qs * HS + qh) * DH + k8);
                        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const float2 f = __bfloat1622float2(p2[x]);
                            acc[2 * x] = f.x;
                            acc[2 * x + 1] = f.y;
                        }
                    }
                    uint4 w;
                    w.x = pack_bf16(acc[0] * a.qscale, acc[1] * a.qscale);
                    w.y = pack_bf16(acc[2] * a.qscale, acc[3] * a.qscale);
                    w.z = pack_bf16(acc[4] * a.qscale, acc[5] * a.qscale);
                    w.w = pack_bf16(acc[6] * a.qscale, acc[7] * a.qscale);
                    *reinterpret_cast<uint4*>(qb + (k8 >> 6) * (HH * 128u) + sw128_offset(h, (k8 & 63) * 2)) = w;
                }
                fence_proxy_async_smem();
                bar_sync(3, NSM);
                if (stid == 0) mbar_arrive(&q_ready[seg & 1]);
#pragma unroll
                for (int h = 0; h < 16; ++h) { m[h] = -INFINITY; lp[h] = 0.f; acc[h] = 0.f; }
            }
            const int j0 = (g - P.tile_prefix[b]) * KT;
            // this group's sequence: the unit's member hg (PAIR), else the tile's sequence
            const int seq = PAIR ? NM * b + hg : b;
            const bool seq_ok = seq < P.batch;
            const int len = seq_ok ? P.len[seq] : 0;
            const bool valid = j0 + jl < len;
            const int s = ks;                    // this tile's K stage and its fill parity
            const uint32_t sph = kph;
            if (++ks == a.ks) { ks = 0; kph ^= 1u; }
            if (!bad) bad = !mbar_wait(&u_full[i & 1], (uint32_t)((i >> 1) & 1), lim, a.err, abort);
            if (!bad) bad = !mbar_wait(&k_full[s], sph, lim, a.err, abort);
            tc_fence_after();
            uint32_t u[16];
            tmem_ld16(lane_addr + (uint32_t)(i & 1) * HH + hbase, u);
            // this row's a^K and a^V for the group's 16 heads
            float ak[16], av[16];
            {
                static_assert(R == 2, "factor words hold both ranks");
                // the 32-bit word holds (head, both ranks); this row's rank picks a half.
                // With the TMA swizzle, 16-byte chunk bits 4..6 are XORed with address bits
                // 7..9 (the tiles are 1024-aligned), so the 16 keys of a warp spread over
                // the banks instead of hitting one or two.
                constexpr uint32_t kRow = HS * R * 2u;
                const uint32_t kSw = a.asw ? 7u : 0u;
                const int ah0 = PAIR ? 0 : hbase;      // the group's first head in the tile
                const uint32_t akr = smem_u32(st_ak(s, PAIR ? hg : 0)) + (uint32_t)jl * kRow;
                const uint32_t avr = smem_u32(st_av(s, PAIR ? hg : 0)) + (uint32_t)jl * kRow;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    uint32_t ka = akr + (uint32_t)(ah0 + h) * 4u, va = avr + (uint32_t)(ah0 + h) * 4u;
                    ka ^= ((ka >> 7) & kSw) << 4;
                    va ^= ((va >> 7) & kSw) << 4;
                    const uint32_t kw = lds_u32(ka);
                    const uint32_t vw = lds_u32(va);
                    ak[h] = sr ? bf16hi(kw) : bf16lo(kw);
                    av[h] = sr ? bf16hi(vw) : bf16lo(vw);
                }
            }
            tmem_ld_wait();
            float sc[16];
            bool over = false;
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                float v = ak[h] * __uint_as_float(u[h]);
#pragma unroll
                for (int o = 1; o < R; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                sc[h] = valid ? v : -INFINITY;
                over |= sc[h] - m[h] > kTau;
            }
            // first tile of a part, or a score above the reference max: exact tile max
            if (bar_any(1 + hg, 128, first || over)) {
                float* rd = red + hg * 192;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    float v = warp_max(sc[h]);
                    if (lane == 0) rd[quarter * 16 + h] = v;
                }
                bar_sync(1 + hg, 128);
                float alpha[16];
                bool resc = false;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    const float mt = fmaxf(fmaxf(rd[h], rd[16 + h]), fmaxf(rd[32 + h], rd[48 + h]));
                    const float mn = fmaxf(m[h], mt);
                    alpha[h] = first ? 1.f : ex2(m[h] - mn);
                    resc |= alpha[h] != 1.f;
                    m[h] = mn;
                    lp[h] *= alpha[h];
                    if constexpr (SB) acc[h] *= alpha[h];
                }
                bar_sync(1 + hg, 128);                 // everyone has read the scratch
                if (!SB && !first && __any_sync(0xffffffffu, resc)) {
                    // O^T columns of this group *= alpha once PV(i-1) has completed
                    if (!bad)
                        bad = !mbar_wait(&w_empty[(i - 1) & 1], (uint32_t)(((i - 1) >> 1) & 1), lim, a.err, abort);
                    tc_fence_after();
                    uint32_t o[16];
                    tmem_ld16(lane_addr + 2u * HH + hbase, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 16; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                    tmem_st16(lane_addr + 2u * HH + hbase, o);
                    tmem_st_wait();
                }
            }
            if constexpr (SB) {
                // shared basis: every value row of rank s is the basis b^V_s, so the
                // values need only sum_j p a^V_{j,h,s}, kept per thread (its row's rank)
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    // (a PAIR member can have no valid key in a whole part: m stays -inf)
                    const float p = valid ? ex2(sc[h] - m[h]) : 0.f;
                    if (sr == 0) lp[h] += p;
                    if (valid) acc[h] = fmaf(p, av[h], acc[h]);   // a^V past the length is not data
                }
            } else {
                // p and W^T (row r = K index, columns = heads), bf16 pairs of adjacent rows
                if (i >= 2 && !bad)
                    bad = !mbar_wait(&w_empty[i & 1], (uint32_t)(((i >> 1) - 1) & 1), lim, a.err, abort);
                uint8_t* wb = wbuf + (size_t)(i & 1) * kQW;
    #pragma unroll
                for (int h = 0; h < 16; ++h) {
                    const float p = ex2(sc[h] - m[h]);
                    if (sr == 0) lp[h] += p;
                    const float w = valid ? p * av[h] : 0.f;
                    const float wn = __shfl_down_sync(0xffffffffu, w, 1);
                    if ((r & 1) == 0) {
                        const int hh = hbase + h;
                        *reinterpret_cast<uint32_t*>(wb + (r >> 6) * (HH * 128u) + sw128_offset(hh, (r & 63) * 2)) =
                            pack_bf16(w, wn);
                    }
                }
                if (hg == 0 && !valid && j0 + jl >= len) {
                    // keys past the sequence: clear their b^V row (once the tile has landed)
                    // so 0 * (cache contents) = 0
                    const int sv = i % kVS;
                    if (!bad) bad = !mbar_wait(&v_full[sv], (uint32_t)((i / kVS) & 1), lim, a.err, abort);
                    if (!bad) {
                        uint4* z0 = reinterpret_cast<uint4*>(st_bv(sv) + r * 128);
                        uint4* z1 = reinterpret_cast<uint4*>(st_bv(sv) + kBox + r * 128);
    #pragma unroll
                        for (int e = 0; e < 8; ++e) { z0[e] = make_uint4(0, 0, 0, 0); z1[e] = make_uint4(0, 0, 0, 0); }
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&w_full[i & 1]);
            mbar_arrive(&k_empty[s]);                // this thread is done with the K stage
            const bool last = (i == n - 1) || (P.tile_prefix[b + 1] <= g + 1);
            if (last) {
                // part done: O^T (lane = d row), l per head, written to the workspace
                // (c_first is per unit; an odd batch's missing member writes nothing)
                const int part = seq_ok ? P.first_part[seq] + (c - P.c_first[b]) : 0;
                if (!in_bounds(!seq_ok || (part >= 0 && part < P.total_parts), a.err)) bad = true;
                const bool wr = seq_ok && !bad;
                const int oh0 = PAIR ? 0 : hbase;        // the group's first head in the sequence
                float* wo = a.ws_o + (size_t)(wr ? part : 0) * HS * DH;
                if constexpr (SB) {
                    // S_{h,s} = sum_j p a^V_{j,h,s}: rows of rank s are the lanes of parity
                    // s (R = 2); sum them in the warp, then over the group's 4 warps, and
                    // O_h = sum_s S_{h,s} b^V_s, one d_h element per thread
                    float* rs = red + hg * 192 + 64;     // [4 warps][R][16]
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        float v = acc[h];
                        v += __shfl_xor_sync(0xffffffffu, v, 2);
                        v += __shfl_xor_sync(0xffffffffu, v, 4);
                        v += __shfl_xor_sync(0xffffffffu, v, 8);
                        v += __shfl_xor_sync(0xffffffffu, v, 16);
                        if (lane < R) rs[(quarter * R + lane) * 16 + h] = v;
                    }
                    bar_sync(1 + hg, 128);
                    if (wr && r < DH) {
                        float bvr[R];
#pragma unroll
                        for (int q = 0; q < R; ++q) bvr[q] = __bfloat162float(a.cb_v[q * DH + r]);
#pragma unroll
                        for (int h = 0; h < 16; ++h) {
                            float o = 0.f;
#pragma unroll
                            for (int q = 0; q < R; ++q) {
                                const float S = (rs[q * 16 + h] + rs[(R + q) * 16 + h]) +
                                                (rs[(2 * R + q) * 16 + h] + rs[(3 * R + q) * 16 + h]);
                                o = fmaf(S, bvr[q], o);
                            }
                            wo[(size_t)(oh0 + h) * DH + r] = o;
                        }
                    }
                } else {
                    if (!bad) bad = !mbar_wait(o_done, (uint32_t)(seg & 1), lim, a.err, abort);
                    tc_fence_after();
                    uint32_t o[16];
                    tmem_ld16(lane_addr + 2u * HH + hbase, o);
                    tmem_ld_wait();
                    if (wr && r < DH) {
#pragma unroll
                        for (int h = 0; h < 16; ++h) wo[(size_t)(oh0 + h) * DH + r] = __uint_as_float(o[h]);
                    }
                }
                float* rd = red + hg * 192;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    const float v = warp_sum(lp[h]);
                    if (lane == 0) rd[quarter * 16 + h] = v;
                }
                bar_sync(1 + hg, 128);
                if (r < 16 && wr) {
                    const float l = (rd[r] + rd[16 + r]) + (rd[32 + r] + rd[48 + r]);
                    a.ws_ml[((size_t)part * HS + oh0 + r) * 2 + 0] = m[r];
                    a.ws_ml[((size_t)part * HS + oh0 + r) * 2 + 1] = l;
                }
                bar_sync(1 + hg, 128);
                if constexpr (!SB) {
                    tc_fence_before();
                    mbar_arrive(o_free);
                }
            }
            if (bar_any(4, NSM, bad)) break;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

template <int DH, int HH, int R, bool SB, bool PAIR>
cudaError_t launch_t(const Shape& s, DecodeTcArgs a, const tpa_cache& c, const DecodePlan& plan,
                     cudaStream_t st) {
    constexpr int KT = 128 / R;
    constexpr int HS = PAIR ? HH / 2 : HH;       // heads per sequence
    constexpr int NM = PAIR ? 2 : 1;             // sequences per tile
    if (PAIR != (plan.pairs != 0)) return cudaErrorInvalidValue;
    a.a_bytes = (uint32_t)(KT * HS * R * 2);
    const uint32_t a_pad = (a.a_bytes + 127u) & ~127u;
    constexpr int NB = DH / 64;
    a.kstage_bytes = ((NB * kBox + 2u * NM * a_pad) + 1023u) & ~1023u;
    // (SB: no V ring, no W^T buffers)
    const size_t fixed = 1024 + (SB ? 0 : (size_t)kVS * 2 * kBox) + (SB ? 2u : 4u) * HH * 256u +
                         (HH / 16) * 192 * sizeof(float) + 32 * 8 + 16;
    a.ks = 4;
    while (a.ks > 2 && fixed + (size_t)a.ks * a.kstage_bytes > 227 * 1024) --a.ks;
    const size_t smem = fixed + (size_t)a.ks * a.kstage_bytes;
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    CUtensorMap tmk, tmv;
    // B rows: every sequence's (contextual), or one per-position table (shared basis)
    const uint64_t dims[2] = {(uint64_t)DH, (uint64_t)(a.bcap ? c.batch : 1) * c.capacity * R};
    const uint64_t stride[1] = {(uint64_t)DH * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_tmap_bf16(&tmk, c.b_k, 2, dims, stride, box) || !make_tmap_bf16(&tmv, c.b_v, 2, dims, stride, box))
        return cudaErrorInvalidValue;
    // a^K, a^V as rows of 128 bytes (h R = 64 bf16: one key at h 32, two keys at h 16),
    // one box of KT keys with the 128-byte swizzle: the per-key reads of unswizzled rows
    // were 16-way (h 32) and 8-way (h 16) bank conflicts.  At h 16 a row holds two keys,
    // so the capacity must be even (else bulk copies).
    constexpr int kpr = 128 / (HS * R * 2);      // keys per 128-byte row
    CUtensorMap tmak, tmav;
    a.asw = (c.capacity % kpr == 0) ? 1 : 0;
    if (a.asw) {
        const uint64_t adims[2] = {64, (uint64_t)c.batch * c.capacity / kpr};
        const uint64_t astride[1] = {128};
        const uint32_t abox[2] = {64, (uint32_t)(KT / kpr)};
        if (!make_tmap_bf16(&tmak, c.a_k, 2, adims, astride, abox) ||
            !make_tmap_bf16(&tmav, c.a_v, 2, adims, astride, abox))
            return cudaErrorInvalidValue;
    } else {
        tmak = tmk;     // unused
        tmav = tmk;
    }
    constexpr int threads = ((HH == 32 && !SB) ? 96 : 128) + 32 * 4 * (HH / 16);
    cudaError_t e = allow_smem(reinterpret_cast<const void*>(decode_tc_kernel<DH, HH, R, SB, PAIR>), (int)smem);
    if (e != cudaSuccess) return e;
    decode_tc_kernel<DH, HH, R, SB, PAIR><<<plan.n_ctas, threads, smem, st>>>(tmk, tmv, tmak, tmav, a, plan);
    return cudaGetLastError();
}
}  // namespace

bool decode_tc_supported(const Shape& s) {
    return s.bf16 && (s.Dh == 64 || s.Dh == 128) && (s.H == 16 || s.H == 32) && s.Rk == 2 &&
           s.Rv == 2 && s.Rq <= 64;
}

cudaError_t launch_decode_tc(const Shape& s, const void* q_a, const void* q_b, const tpa_cache& c,
                             const DecodePlan& plan, float* ws, int* err, uint32_t wait_limit,
                             cudaStream_t st) {
    if ((long long)c.batch * c.capacity * s.Rk >= (1LL << 31)) return cudaErrorInvalidValue;
    if (plan.total_tiles < 1 || plan.n_ctas < 1) return cudaErrorInvalidValue;
    DecodeTcArgs a{};
    a.q_a = static_cast<const __nv_bfloat16*>(q_a);
    a.q_b = static_cast<const __nv_bfloat16*>(q_b);
    a.ca_k = static_cast<const __nv_bfloat16*>(c.a_k);
    a.ca_v = static_cast<const __nv_bfloat16*>(c.a_v);
    a.ws_ml = ws;
    a.ws_o = ws + (size_t)plan.total_parts * s.H * 2;
    a.Rq = s.Rq;
    a.cap = c.capacity;
    a.bcap = (int)b_seq_rows(s, c);
    a.cache_batch = c.batch;
    a.qscale = 1.4426950408889634f / ((s.Rq > 0 ? (float)s.Rq : 1.f) * (float)s.Rk * std::sqrt((float)s.Dh));
    a.err = err;
    a.wait_limit = wait_limit;
    a.cb_v = static_cast<const __nv_bfloat16*>(c.b_v);
    if (s.shared) {
        // h 16: two sequences per key tile (32 score columns), sharing its table tile
        if (s.Dh == 64) return s.H == 16 ? launch_t<64, 32, 2, true, true>(s, a, c, plan, st)
                                         : launch_t<64, 32, 2, true, false>(s, a, c, plan, st);
        return s.H == 16 ? launch_t<128, 32, 2, true, true>(s, a, c, plan, st)
                         : launch_t<128, 32, 2, true, false>(s, a, c, plan, st);
    }
    if (s.Dh == 64) return s.H == 16 ? launch_t<64, 16, 2, false, false>(s, a, c, plan, st)
                                     : launch_t<64, 32, 2, false, false>(s, a, c, plan, st);
    return s.H == 16 ? launch_t<128, 16, 2, false, false>(s, a, c, plan, st)
                     : launch_t<128, 32, 2, false, false>(s, a, c, plan, st);
}

}  // namespace tpa
