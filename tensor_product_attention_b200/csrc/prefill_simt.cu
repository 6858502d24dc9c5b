// Causal prefill from factors on the CUDA cores (fp32), used for fp32 layers.
//
// One warp per (token, head).  The warp folds the query factors into the head's query
// q_h = (1/R_Q) sum_r a^Q_{h,r} b^Q_r once, then walks the cached keys j <= position,
// scoring each as (1/R_K) sum_s a^K_{j,h,s} (q_h . b^K_{j,s}) / sqrt(d_h) and adding
// (1/R_V) sum_s a^V_{j,h,s} b^V_{j,s} under an online softmax.  K and V are formed
// one key at a time in registers and never stored.  Formulas: "【拜读】Tensor Product
// Attention Is All You Need…" (coreui.cn), §3 公式描述 and 代码 前向传播; attention per
// the jieyibu.net TPA page, Ⅱ.1.
#include "tpa_internal.h"
#include "device_util.cuh"

namespace tpa {

namespace {
constexpr int MAXU = 8;   // head_dim <= 256

struct PrefillArgs {
    const void *a_q, *b_q;
    const void *ca_k, *ca_v, *cb_k, *cb_v;
    void* out;
    int T, S, H, Dh, Rq, Rk, Rv, cap;
    long long bcap;       // B_K / B_V rows between sequences: cap, or 0 (shared basis)
    int cache_batch;      // sequences the cache holds (bounds checks)
    int* err;
};

template <typename T>
__global__ void __launch_bounds__(128) prefill_simt_kernel(PrefillArgs a, SeqParams start) {
    const int lane = threadIdx.x & 31;
    const long long warp = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
    if (warp >= (long long)a.T * a.H) return;
    const int t = (int)(warp / a.H), h = (int)(warp % a.H);
    const int b = t / a.S, i = t - b * a.S;
    const int pos = start.v[b] + i;
    // every cache row this warp reads is (b, j <= pos)
    if (!in_bounds(b < a.cache_batch && pos < a.cap, a.err)) return;
    const T* aq = reinterpret_cast<const T*>(a.a_q);
    const T* bq = reinterpret_cast<const T*>(a.b_q);
    const T* ak = reinterpret_cast<const T*>(a.ca_k);
    const T* av = reinterpret_cast<const T*>(a.ca_v);
    const T* bk = reinterpret_cast<const T*>(a.cb_k);
    const T* bv = reinterpret_cast<const T*>(a.cb_v);

    // TPA-KVonly (Rq = 0): the query row is given, q_{t,h} = b_q[t][h][:]
    const float qscale = kLog2e / ((float)(a.Rq > 0 ? a.Rq : 1) * (float)a.Rk * sqrtf((float)a.Dh));
    float q[MAXU], acc[MAXU];
#pragma unroll
    for (int u = 0; u < MAXU; ++u) {
        int e = lane + 32 * u;
        float v = 0.f;
        if (e < a.Dh) {
            if (a.Rq == 0)
                v = to_f(bq[((long long)t * a.H + h) * a.Dh + e]);
            for (int r = 0; r < a.Rq; ++r)
                v = fmaf(to_f(aq[((long long)t * a.H + h) * a.Rq + r]),
                         to_f(bq[((long long)t * a.Rq + r) * a.Dh + e]), v);
        }
        q[u] = v * qscale;
        acc[u] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    const long long seq_row = (long long)b * a.cap, bseq_row = (long long)b * a.bcap;
    for (int j = 0; j <= pos; ++j) {
        const long long row = seq_row + j, brow = bseq_row + j;
        float s = 0.f;
        for (int sk = 0; sk < a.Rk; ++sk) {
            float dot = 0.f;
#pragma unroll
            for (int u = 0; u < MAXU; ++u) {
                int e = lane + 32 * u;
                if (e < a.Dh) dot = fmaf(q[u], to_f(bk[(brow * a.Rk + sk) * a.Dh + e]), dot);
            }
            dot = warp_sum(dot);
            s = fmaf(to_f(ak[(row * a.H + h) * a.Rk + sk]), dot, s);
        }
        const float m_new = fmaxf(m, s);
        const float alpha = exp2f(m - m_new);
        const float p = exp2f(s - m_new);
        l = l * alpha + p;
        m = m_new;
#pragma unroll
        for (int u = 0; u < MAXU; ++u) {
            int e = lane + 32 * u;
            float v = 0.f;
            if (e < a.Dh)
                for (int sv = 0; sv < a.Rv; ++sv)
                    v = fmaf(to_f(av[(row * a.H + h) * a.Rv + sv]),
                             to_f(bv[(brow * a.Rv + sv) * a.Dh + e]), v);
            acc[u] = fmaf(acc[u], alpha, p * v);
        }
    }
    T* out = reinterpret_cast<T*>(a.out);
    const float inv = 1.f / (l * (float)a.Rv);
#pragma unroll
    for (int u = 0; u < MAXU; ++u) {
        int e = lane + 32 * u;
        if (e < a.Dh) out[((long long)t * a.H + h) * a.Dh + e] = from_f<T>(acc[u] * inv);
    }
}
}  // namespace

cudaError_t launch_prefill_simt(const Shape& s, const tpa_factors& q, const tpa_cache& c,
                                int batch, int seqlen, const SeqParams& start, void* out,
                                int* err, cudaStream_t st) {
    PrefillArgs a;
    a.cache_batch = c.batch;
    a.err = err;
    a.a_q = q.a_q; a.b_q = q.b_q;
    a.ca_k = c.a_k; a.ca_v = c.a_v; a.cb_k = c.b_k; a.cb_v = c.b_v;
    a.out = out;
    a.T = batch * seqlen; a.S = seqlen; a.H = s.H; a.Dh = s.Dh;
    a.Rq = s.Rq; a.Rk = s.Rk; a.Rv = s.Rv; a.cap = c.capacity; a.bcap = b_seq_rows(s, c);
    long long warps = (long long)a.T * a.H;
    long long blocks = (warps * 32 + 127) / 128;
    if (s.bf16)
        prefill_simt_kernel<__nv_bfloat16><<<(unsigned)blocks, 128, 0, st>>>(a, start);
    else
        prefill_simt_kernel<float><<<(unsigned)blocks, 128, 0, st>>>(a, start);
    return cudaGetLastError();
}

}  // namespace tpa
