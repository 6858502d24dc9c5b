// Decode from the factor cache on the CUDA cores (fp32 layers), the split schedule,
// and the split-merge ("combine") kernel shared by every decode kernel.
//
// One query per sequence at position len-1 attends to cached keys 0..len-1 ("【拜读】
// Tensor Product Attention Is All You Need…" (coreui.cn), 代码 前向传播: the cache is
// written, then read over [:start_pos+seqlen]).  B_K is used as cached, already rotated
// (same page, 关键问题及回答 问题2), so decode applies no RoPE.  The query is folded once
// per sequence, q_h = (1/R_Q) sum_r a^Q_{h,r} b^Q_r (or given, TPA-KVonly); each key
// then costs h*R_K*d_h multiply-adds for the scores and h*R_V*d_h for the values.
//
// Split-K over the context: CTA (split, b) walks keys [split*split_len, ...) and writes
// its partial softmax state (running max m, sum l, unnormalised o) to the workspace;
// the combine kernel merges the splits of a sequence in increasing split order, so
// the result does not depend on scheduling.
#include <algorithm>

#include "tpa_internal.h"
#include "device_util.cuh"
#include "tmap.h"

namespace tpa {

// Paired plan: unit u = sequences (2u, 2u+1) (the last unit of an odd batch has one);
// its tiles cover the longer member.  The CTAs c_first[u] .. c_first[u] + n - 1 that
// overlap the unit give member 0 parts base .. base+n-1 and member 1 parts
// base+n .. base+2n-1, so each sequence's parts stay consecutive for the merge.
static void make_paired_plan(const int32_t* lengths, int batch, int kt, DecodePlan* plan) {
    DecodePlan& P = *plan;
    const int U = (batch + 1) / 2;
    P.n_units = U;
    long long n = 0;
    for (int u = 0; u < U; ++u) {
        P.tile_prefix[u] = (int32_t)n;
        const int len = std::max(lengths[2 * u], 2 * u + 1 < batch ? lengths[2 * u + 1] : 0);
        n += (len + kt - 1) / kt;
    }
    P.tile_prefix[U] = (int32_t)n;
    P.total_tiles = (int32_t)n;
    const int G = (int)std::min<long long>(sm_count(), n);
    P.n_ctas = G;
    int32_t n_cta[TPA_MAX_BATCH];
    for (int u = 0; u < U; ++u) n_cta[u] = 0;
    int u = 0;
    for (int c = 0; c < G; ++c) {
        const long long lo = c * n / G, hi = (c + 1) * n / G;
        while (u < U && P.tile_prefix[u + 1] <= lo) ++u;
        for (int uu = u; uu < U && P.tile_prefix[uu] < hi; ++uu) {
            if (P.tile_prefix[uu + 1] <= lo) continue;
            if (n_cta[uu] == 0) P.c_first[uu] = c;
            ++n_cta[uu];
        }
    }
    int part = 0;
    for (int v = 0; v < U; ++v) {
        for (int m = 0; m < 2; ++m) {
            const int b = 2 * v + m;
            if (b >= batch) break;
            P.first_part[b] = part;
            P.n_parts[b] = n_cta[v];
            part += n_cta[v];
        }
    }
    P.total_parts = part;
}

void make_decode_plan(const Shape& s, const int32_t* lengths, int batch, bool tc,
                      DecodePlan* plan) {
    DecodePlan& P = *plan;
    P.batch = batch;
    P.pairs = 0;
    P.n_units = batch;
    long long total = 0;
    for (int b = 0; b < batch; ++b) {
        P.len[b] = lengths[b];
        total += lengths[b];
    }
    if (!tc) {
        // splits of split_len keys (a multiple of 128), about 4 CTAs per SM in all
        const int tile = 128;
        const long long target_ctas = (long long)sm_count() * 4;
        const long long per = (total + target_ctas - 1) / target_ctas;
        P.split_len = (int)std::max<long long>(tile, ((per + tile - 1) / tile) * tile);
        P.key_tile = tile;
        int part = 0, max_splits = 1;
        for (int b = 0; b < batch; ++b) {
            P.first_part[b] = part;
            P.n_parts[b] = (lengths[b] + P.split_len - 1) / P.split_len;
            part += P.n_parts[b];
            max_splits = std::max(max_splits, (int)P.n_parts[b]);
        }
        P.total_parts = part;
        P.n_ctas = max_splits;          // grid.x of the split kernel
        P.total_tiles = 0;
        return;
    }
    // persistent grid over the concatenated key tiles of all sequences (or units)
    const int kt = 128 / s.Rk;
    P.key_tile = kt;
    P.split_len = 0;
    P.pairs = decode_pairs(s) ? 1 : 0;
    if (P.pairs) {
        make_paired_plan(lengths, batch, kt, &P);
        return;
    }
    P.n_units = batch;
    long long n = 0;
    for (int b = 0; b < batch; ++b) {
        P.tile_prefix[b] = (int32_t)n;
        n += (lengths[b] + kt - 1) / kt;
    }
    P.tile_prefix[batch] = (int32_t)n;
    P.total_tiles = (int32_t)n;
    const int G = (int)std::min<long long>(sm_count(), n);
    P.n_ctas = G;
    auto g0 = [&](long long c) { return c * n / G; };
    // parts in (CTA, sequence) order; the parts of one sequence are consecutive
    int part = 0;
    int b = 0;
    for (int b2 = 0; b2 < batch; ++b2) P.n_parts[b2] = 0;
    for (int c = 0; c < G; ++c) {
        const long long lo = g0(c), hi = g0(c + 1);
        while (b < batch && P.tile_prefix[b + 1] <= lo) ++b;
        for (int bb = b; bb < batch && P.tile_prefix[bb] < hi; ++bb) {
            if (P.tile_prefix[bb + 1] <= lo) continue;
            if (P.n_parts[bb] == 0) {
                P.first_part[bb] = part;
                P.c_first[bb] = c;
            }
            ++P.n_parts[bb];
            ++part;
        }
    }
    P.total_parts = part;
}

size_t decode_workspace_bytes(const Shape& s, const DecodePlan& plan) {
    return (size_t)plan.total_parts * s.H * (2 + (size_t)s.Dh) * sizeof(float);
}

namespace {
constexpr int KT = 32;     // keys per shared-memory tile
constexpr int NT = 256;    // threads per CTA
constexpr int MAXO = 32;   // output elements per thread: h*d_h <= 8192

struct DecodeArgs {
    const void *q_a, *q_b;
    const void *ca_k, *ca_v, *cb_k, *cb_v;
    float* ws_ml;   // [parts][H][2]
    float* ws_o;    // [parts][H][Dh]
    int H, Dh, Rq, Rk, Rv, cap, split_len;
    long long bcap;   // B_K / B_V rows between sequences: cap, or 0 (shared basis)
    int cache_batch;  // sequences the cache holds (bounds checks)
    int* err;
};

template <typename T>
__global__ void __launch_bounds__(NT) decode_simt_kernel(DecodeArgs a, const DecodePlan plan) {
    const int split = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int L = plan.len[b];
    const int j0 = split * a.split_len;
    if (j0 >= L) return;
    const int j1 = min(L, j0 + a.split_len);
    // every cache row this CTA reads is (b, j < L); its part slot must exist
    if (!in_bounds(b < a.cache_batch && L <= a.cap && plan.first_part[b] + split < plan.total_parts, a.err))
        return;
    const int H = a.H, Dh = a.Dh;
    const int bk_row = a.Rk * Dh + 1;   // padded per-key stride: conflict-free score loop

    extern __shared__ float sm[];
    float* qs = sm;                          // [H][Dh] scaled query
    float* bks = qs + H * Dh;                // [KT][bk_row]
    float* bvs = bks + KT * bk_row;          // [KT][Rv][Dh]
    float* akT = bvs + KT * a.Rv * Dh;       // [H*Rk][KT]
    float* avT = akT + H * a.Rk * KT;        // [H*Rv][KT]
    float* sc = avT + H * a.Rv * KT;         // [H][KT]
    float* mrow = sc + H * KT;               // [H]
    float* lrow = mrow + H;                  // [H]
    float* alph = lrow + H;                  // [H]

    const T* qa = reinterpret_cast<const T*>(a.q_a);
    const T* qb = reinterpret_cast<const T*>(a.q_b);
    const float scale = kLog2e / ((float)a.Rk * sqrtf((float)Dh));
    for (int idx = tid; idx < H * Dh; idx += NT) {
        int h = idx / Dh, e = idx - h * Dh;
        float v;
        if (a.Rq > 0) {
            v = 0.f;
            for (int r = 0; r < a.Rq; ++r)
                v = fmaf(to_f(qa[((long long)b * H + h) * a.Rq + r]),
                         to_f(qb[((long long)b * a.Rq + r) * Dh + e]), v);
            v /= (float)a.Rq;
        } else {
            v = to_f(qb[((long long)b * H + h) * Dh + e]);
        }
        qs[idx] = v * scale;
    }
    for (int h = tid; h < H; h += NT) { mrow[h] = -INFINITY; lrow[h] = 0.f; }
    float acc[MAXO];
#pragma unroll
    for (int u = 0; u < MAXO; ++u) acc[u] = 0.f;

    const T* ak = reinterpret_cast<const T*>(a.ca_k);
    const T* av = reinterpret_cast<const T*>(a.ca_v);
    const T* bk = reinterpret_cast<const T*>(a.cb_k);
    const T* bv = reinterpret_cast<const T*>(a.cb_v);
    const long long seq_row = (long long)b * a.cap, bseq_row = (long long)b * a.bcap;

    for (int jt = j0; jt < j1; jt += KT) {
        const int n = min(KT, j1 - jt);
        __syncthreads();
        for (int u = tid; u < n * a.Rk * Dh; u += NT) {
            int j = u / (a.Rk * Dh), r = u - j * (a.Rk * Dh);
            bks[j * bk_row + r] = to_f(bk[(bseq_row + jt) * a.Rk * Dh + u]);
        }
        for (int u = tid; u < n * a.Rv * Dh; u += NT)
            bvs[u] = to_f(bv[(bseq_row + jt) * a.Rv * Dh + u]);
        for (int u = tid; u < n * H * a.Rk; u += NT) {
            int j = u / (H * a.Rk), hr = u - j * (H * a.Rk);
            akT[hr * KT + j] = to_f(ak[(seq_row + jt) * H * a.Rk + u]);
        }
        for (int u = tid; u < n * H * a.Rv; u += NT) {
            int j = u / (H * a.Rv), hr = u - j * (H * a.Rv);
            avT[hr * KT + j] = to_f(av[(seq_row + jt) * H * a.Rv + u]);
        }
        __syncthreads();
        // scores, log2 domain
        for (int u = tid; u < H * KT; u += NT) {
            int h = u / KT, j = u - h * KT;
            float s = -INFINITY;
            if (j < n) {
                s = 0.f;
                for (int sk = 0; sk < a.Rk; ++sk) {
                    const float* kr = bks + j * bk_row + sk * Dh;
                    const float* qr = qs + h * Dh;
                    float dot = 0.f;
                    for (int e = 0; e < Dh; ++e) dot = fmaf(qr[e], kr[e], dot);
                    s = fmaf(akT[(h * a.Rk + sk) * KT + j], dot, s);
                }
            }
            sc[u] = s;
        }
        __syncthreads();
        for (int h = tid; h < H; h += NT) {
            float mt = -INFINITY;
            for (int j = 0; j < n; ++j) mt = fmaxf(mt, sc[h * KT + j]);
            float m_new = fmaxf(mrow[h], mt);
            float alpha = exp2f(mrow[h] - m_new);
            float sum = 0.f;
            for (int j = 0; j < KT; ++j) {
                float p = (j < n) ? exp2f(sc[h * KT + j] - m_new) : 0.f;
                sc[h * KT + j] = p;
                sum += p;
            }
            lrow[h] = lrow[h] * alpha + sum;
            mrow[h] = m_new;
            alph[h] = alpha;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < MAXO; ++u) {
            int idx = tid + NT * u;
            if (idx < H * Dh) {
                int h = idx / Dh, e = idx - h * Dh;
                float v = acc[u] * alph[h];
                for (int j = 0; j < n; ++j) {
                    float vj = 0.f;
                    for (int sv = 0; sv < a.Rv; ++sv)
                        vj = fmaf(avT[(h * a.Rv + sv) * KT + j], bvs[(j * a.Rv + sv) * Dh + e], vj);
                    v = fmaf(sc[h * KT + j], vj, v);
                }
                acc[u] = v;
            }
        }
    }
    __syncthreads();
    const long long part = (long long)(plan.first_part[b] + split) * H;
    for (int h = tid; h < H; h += NT) {
        a.ws_ml[(part + h) * 2 + 0] = mrow[h];
        a.ws_ml[(part + h) * 2 + 1] = lrow[h];
    }
#pragma unroll
    for (int u = 0; u < MAXO; ++u) {
        int idx = tid + NT * u;
        if (idx < H * Dh) a.ws_o[part * Dh + idx] = acc[u];
    }
}

struct CombineArgs {
    const float* ws_ml;
    const float* ws_o;
    void* out;
    int H, Dh, Rv;
    int* err;
};

// grid (H, batch), one thread per output element of the head.  Parts are merged in
// increasing part order, so the result does not depend on scheduling.
template <typename T>
__global__ void decode_combine_kernel(CombineArgs a, const DecodePlan plan) {
    const int h = blockIdx.x, b = blockIdx.y;
    const int nsplit = plan.n_parts[b];
    const long long base = plan.first_part[b];
    if (!in_bounds(base >= 0 && base + nsplit <= plan.total_parts, a.err)) return;
    float m = -INFINITY;
    for (int k = 0; k < nsplit; ++k) m = fmaxf(m, a.ws_ml[((base + k) * a.H + h) * 2]);
    float den = 0.f;
    for (int k = 0; k < nsplit; ++k) {
        const float* ml = a.ws_ml + ((base + k) * a.H + h) * 2;
        den = fmaf(exp2f(ml[0] - m), ml[1], den);
    }
    const float inv = 1.f / (den * (float)a.Rv);
    T* out = reinterpret_cast<T*>(a.out);
    for (int e = threadIdx.x; e < a.Dh; e += blockDim.x) {
        float num = 0.f;
        for (int k = 0; k < nsplit; ++k) {
            float wgt = exp2f(a.ws_ml[((base + k) * a.H + h) * 2] - m);
            num = fmaf(wgt, a.ws_o[((base + k) * a.H + h) * (long long)a.Dh + e], num);
        }
        out[((long long)b * a.H + h) * a.Dh + e] = from_f<T>(num * inv);
    }
}
}  // namespace

static size_t decode_simt_smem(const Shape& s) {
    int bk_row = s.Rk * s.Dh + 1;
    size_t fl = (size_t)s.H * s.Dh + (size_t)KT * bk_row + (size_t)KT * s.Rv * s.Dh +
                (size_t)s.H * (s.Rk + s.Rv) * KT + (size_t)s.H * KT + 3 * (size_t)s.H;
    return fl * sizeof(float);
}

cudaError_t launch_decode_simt(const Shape& s, const void* q_a, const void* q_b,
                               const tpa_cache& c, const DecodePlan& plan, float* ws, int* err,
                               cudaStream_t st) {
    if ((long long)s.H * s.Dh > (long long)NT * MAXO) return cudaErrorInvalidValue;
    DecodeArgs a;
    a.cache_batch = c.batch;
    a.err = err;
    a.q_a = q_a; a.q_b = q_b;
    a.ca_k = c.a_k; a.ca_v = c.a_v; a.cb_k = c.b_k; a.cb_v = c.b_v;
    a.ws_ml = ws;
    a.ws_o = ws + (size_t)plan.total_parts * s.H * 2;
    a.H = s.H; a.Dh = s.Dh; a.Rq = s.Rq; a.Rk = s.Rk; a.Rv = s.Rv; a.cap = c.capacity;
    a.bcap = b_seq_rows(s, c);
    a.split_len = plan.split_len;
    size_t smem = decode_simt_smem(s);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    dim3 grid(plan.n_ctas, plan.batch);
    cudaError_t e;
    if (s.bf16) {
        e = allow_smem(reinterpret_cast<const void*>(decode_simt_kernel<__nv_bfloat16>), (int)smem);
        if (e != cudaSuccess) return e;
        decode_simt_kernel<__nv_bfloat16><<<grid, NT, smem, st>>>(a, plan);
    } else {
        e = allow_smem(reinterpret_cast<const void*>(decode_simt_kernel<float>), (int)smem);
        if (e != cudaSuccess) return e;
        decode_simt_kernel<float><<<grid, NT, smem, st>>>(a, plan);
    }
    return cudaGetLastError();
}

cudaError_t launch_decode_combine(const Shape& s, const DecodePlan& plan, const float* ws,
                                  void* out, int* err, cudaStream_t st) {
    CombineArgs a;
    a.err = err;
    a.ws_ml = ws;
    a.ws_o = ws + (size_t)plan.total_parts * s.H * 2;
    a.out = out;
    a.H = s.H; a.Dh = s.Dh; a.Rv = s.Rv;
    dim3 grid(s.H, plan.batch);
    int threads = std::min(256, ((s.Dh + 31) / 32) * 32);
    if (s.bf16)
        decode_combine_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(a, plan);
    else
        decode_combine_kernel<float><<<grid, threads, 0, st>>>(a, plan);
    return cudaGetLastError();
}

}  // namespace tpa
