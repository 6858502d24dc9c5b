// Factor projection on the CUDA cores (fp32 FMA), used for fp32 layers.
//
// Y[T][N] = x[T][D] W_cat[N][D]^T, the six bias-free projections of the TPA module
// ("【拜读】Tensor Product Attention Is All You Need…" (coreui.cn), 代码 类定义与初始化 and
// 前向传播) as one GEMM, with RoPE applied in the epilogue to the B_Q and B_K columns
// (B_K rotated before it is cached, same page, 关键问题及回答 问题2).  fp32 inputs keep
// fp32 accuracy end to end, which the tensor-core path (TF32 at best) would not.
#include "tpa_internal.h"
#include "device_util.cuh"

namespace tpa {

namespace {
constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

struct ProjArgs {
    const void* x;
    const void* w;
    int T, N, D, seqlen, Dh;
    const float2* cs;
    ProjLayout L;
    int* err;
};

__device__ __forceinline__ int segment_of(const ProjLayout& L, int c) {
    int s = 0;
#pragma unroll
    for (int i = 1; i < 6; ++i) s += (c >= L.off[i]);
    return s;
}

template <typename T>
__device__ __forceinline__ void store_col(const ProjLayout& L, int seg, int t, long long tkv, int c, float v,
                                          int* err) {
    int width = L.off[seg + 1] - L.off[seg];
    T* dst = reinterpret_cast<T*>(L.dst[seg]);
    const long long row = seg_row(L, seg, t, tkv);
    if (in_bounds(row >= 0 && row < L.rows[seg] && c - L.off[seg] < width, err))
        dst[row * width + (c - L.off[seg])] = from_f<T>(v);
}

template <typename T>
__global__ void __launch_bounds__(NT) project_simt_kernel(ProjArgs a, SeqParams start) {
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    const T* __restrict__ x = reinterpret_cast<const T*>(a.x);
    const T* __restrict__ w = reinterpret_cast<const T*>(a.w);
    const int tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    const int row0 = blockIdx.y * BM, col0 = blockIdx.x * BN;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < a.D; k0 += BK) {
        for (int u = tid; u < BM * BK; u += NT) {
            int r = u / BK, kk = u % BK;
            int gr = row0 + r, gk = k0 + kk;
            As[kk][r] = (gr < a.T && gk < a.D) ? to_f(x[(long long)gr * a.D + gk]) : 0.f;
            int gc = col0 + r;
            Bs[kk][r] = (gc < a.N && gk < a.D) ? to_f(w[(long long)gc * a.D + gk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    // epilogue: split into the six factors, rotate B_Q / B_K pairs
    const ProjLayout& L = a.L;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int t = row0 + ty * 4 + i;
        if (t >= a.T) continue;
        int b = t / a.seqlen;
        int pos = start.v[b] + (t - b * a.seqlen);
        const long long tkv = (long long)b * L.kv_cap + pos;
        // cache mode: the sequence's last token records the new length, once
        if (L.lengths && col0 == 0 && tx == 0 && t - b * a.seqlen == a.seqlen - 1 &&
            in_bounds(b < L.n_lengths, a.err))
            L.lengths[b] = pos + 1;
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) {
            int c = col0 + tx * 4 + 2 * jp;
            if (c >= a.N) continue;
            int seg = segment_of(L, c);
            float y0 = acc[i][2 * jp], y1 = acc[i][2 * jp + 1];
            if (seg == 3 || seg == 4) {
                // segment starts are even, so (c, c+1) is one RoPE pair (2k, 2k+1)
                int local = c - L.off[seg];
                int k2 = (local % a.Dh) >> 1;
                float2 r = make_float2(1.f, 0.f);
                if (in_bounds(pos < L.cs_rows, a.err)) r = a.cs[(long long)pos * (a.Dh >> 1) + k2];
                store_col<T>(L, seg, t, tkv, c, y0 * r.x - y1 * r.y, a.err);
                store_col<T>(L, seg, t, tkv, c + 1, y0 * r.y + y1 * r.x, a.err);
            } else {
                store_col<T>(L, seg, t, tkv, c, y0, a.err);
                if (c + 1 < a.N) store_col<T>(L, segment_of(L, c + 1), t, tkv, c + 1, y1, a.err);
            }
        }
    }
}
}  // namespace

cudaError_t launch_project_simt(const Shape& s, const void* x, const void* w, int batch,
                                int seqlen, const SeqParams& start, const float* cs,
                                const ProjLayout& L, int* err, cudaStream_t st) {
    ProjArgs a;
    a.err = err;
    a.x = x; a.w = w; a.T = batch * seqlen; a.N = L.off[6]; a.D = s.D; a.seqlen = seqlen;
    a.Dh = s.Dh; a.cs = reinterpret_cast<const float2*>(cs); a.L = L;
    dim3 grid((a.N + BN - 1) / BN, (a.T + BM - 1) / BM);
    if (s.bf16)
        project_simt_kernel<__nv_bfloat16><<<grid, NT, 0, st>>>(a, start);
    else
        project_simt_kernel<float><<<grid, NT, 0, st>>>(a, start);
    return cudaGetLastError();
}

}  // namespace tpa
