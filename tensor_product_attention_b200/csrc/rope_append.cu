// RoPE table and factor-cache append.
//
// RoPE table: the caller-supplied freqs_cis of the TPA forward(x, start_pos, freqs_cis,
// mask) in "【拜读】Tensor Product Attention Is All You Need…" (coreui.cn), 代码 前向传播,
// laid out as cs[p][k] = (cos, sin)(p * base^(-2k/d_h)); angles in fp64 so that
// positions up to 2^17 keep full fp32 accuracy.
//
// Cache append: cache[:bsz, start_pos:start_pos+seqlen] = factors from the same forward,
// done as one bit-exact, 16-byte vectorised, coalesced copy of the four cached factor
// tensors; HBM-bound (reads and writes (R_K+R_V)(h+d_h) elements per token).
#include "tpa_internal.h"
#include "device_util.cuh"

namespace tpa {

__global__ void rope_table_kernel(float2* __restrict__ cs, int max_pos, int half,
                                  int head_dim, double base) {
    long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= (long long)max_pos * half) return;
    int p = (int)(idx / half);
    int k = (int)(idx % half);
    double theta = pow(base, -2.0 * (double)k / (double)head_dim);
    double s, c;
    sincos((double)p * theta, &s, &c);
    cs[idx] = make_float2((float)c, (float)s);
}

cudaError_t launch_rope_table(float* cs, int max_pos, int head_dim, double base,
                              cudaStream_t st) {
    int half = head_dim / 2;
    long long n = (long long)max_pos * half;
    int threads = 256;
    long long blocks = (n + threads - 1) / threads;
    rope_table_kernel<<<(unsigned)blocks, threads, 0, st>>>(reinterpret_cast<float2*>(cs),
                                                            max_pos, half, head_dim, base);
    return cudaGetLastError();
}

struct AppendArgs {
    const char* src[4];
    char* dst[4];
    long long row_units[4];   // units of V per token row
    int batch, n_tokens, capacity;
    int32_t* lengths;
};

// grid.y selects one of the four cached tensors; grid.x strides over its rows.
template <typename V>
__global__ void append_kernel(AppendArgs a, SeqParams start) {
    if (blockIdx.x == 0 && blockIdx.y == 0) {
        for (int b = threadIdx.x; b < a.batch; b += blockDim.x)
            a.lengths[b] = start.v[b] + a.n_tokens;
    }
    const int arr = blockIdx.y;
    const long long ru = a.row_units[arr];
    const V* __restrict__ src = reinterpret_cast<const V*>(a.src[arr]);
    V* __restrict__ dst = reinterpret_cast<V*>(a.dst[arr]);
    const long long total = (long long)a.batch * a.n_tokens * ru;
    for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < total;
         u += (long long)gridDim.x * blockDim.x) {
        long long tok = u / ru;
        long long e = u - tok * ru;
        int b = (int)(tok / a.n_tokens);
        int i = (int)(tok - (long long)b * a.n_tokens);
        long long row = (long long)b * a.capacity + start.v[b] + i;
        dst[row * ru + e] = src[u];
    }
}

cudaError_t launch_cache_append(const Shape& s, const tpa_cache& c, const tpa_factors& kv,
                                int batch, int n_tokens, const SeqParams& start,
                                cudaStream_t st) {
    const int es = s.bf16 ? 2 : 4;
    long long row_bytes[4] = {(long long)s.H * s.Rk * es, (long long)s.H * s.Rv * es,
                              (long long)s.Rk * s.Dh * es, (long long)s.Rv * s.Dh * es};
    // widest vector that divides every row (pointers are 16-byte aligned by contract)
    int vec = 16;
    for (int i = 0; i < 4; ++i)
        while (row_bytes[i] % vec) vec >>= 1;
    AppendArgs a;
    a.src[0] = (const char*)kv.a_k; a.src[1] = (const char*)kv.a_v;
    a.src[2] = (const char*)kv.b_k; a.src[3] = (const char*)kv.b_v;
    a.dst[0] = (char*)c.a_k; a.dst[1] = (char*)c.a_v;
    a.dst[2] = (char*)c.b_k; a.dst[3] = (char*)c.b_v;
    for (int i = 0; i < 4; ++i) a.row_units[i] = row_bytes[i] / vec;
    a.batch = batch; a.n_tokens = n_tokens; a.capacity = c.capacity; a.lengths = c.lengths;
    long long most = 0;
    for (int i = 0; i < 4; ++i) {
        long long t = (long long)batch * n_tokens * a.row_units[i];
        if (t > most) most = t;
    }
    int threads = 256;
    long long blocks = (most + threads - 1) / threads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    dim3 grid((unsigned)blocks, 4);
    switch (vec) {
        case 16: append_kernel<uint4><<<grid, threads, 0, st>>>(a, start); break;
        case 8: append_kernel<uint2><<<grid, threads, 0, st>>>(a, start); break;
        case 4: append_kernel<uint32_t><<<grid, threads, 0, st>>>(a, start); break;
        default: append_kernel<uint16_t><<<grid, threads, 0, st>>>(a, start); break;
    }
    return cudaGetLastError();
}

}  // namespace tpa
