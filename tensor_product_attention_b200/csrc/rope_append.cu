// RoPE table and factor-cache append.
//
// RoPE table: the caller-supplied freqs_cis of the TPA forward(x, start_pos, freqs_cis,
// mask) in "【拜读】Tensor Product Attention Is All You Need…" (coreui.cn), 代码 前向传播,
// laid out as cs[p][k] = (cos, sin)(p * base^(-2k/d_h)); angles in fp64 so that
// positions up to 2^17 keep full fp32 accuracy.
//
// Cache append: cache[:bsz, start_pos:start_pos+seqlen] = factors from the same forward,
// done as one bit-exact, 16-byte vectorised, coalesced copy of the four cached factor
// tensors; HBM-bound (reads and writes (R_K+R_V)(h+d_h) elements per token).  With a
// shared basis only A_K and A_V are per token, so only those two are copied.
//
// Shared-basis tables: the variant that shares the basis vectors across tokens (same
// page, 优点与创新 5) keeps B_K and B_V as layer parameters.  Its cache side is one
// table per layer, row p = the key basis rotated at position p (pre-rotated as B_K is
// cached, 关键问题及回答 问题2) and the value basis, which every sequence reads.
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
    long long dst_rows;      // cache rows (batch * capacity): bounds checks
    int n_lengths;
    int* err;
};

// grid.y selects one of the four cached tensors; grid.x strides over its rows.
template <typename V>
__global__ void append_kernel(AppendArgs a, SeqParams start) {
    if (blockIdx.x == 0 && blockIdx.y == 0) {
        for (int b = threadIdx.x; b < a.batch; b += blockDim.x)
            if (in_bounds(b < a.n_lengths, a.err)) a.lengths[b] = start.v[b] + a.n_tokens;
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
        if (in_bounds(row < a.dst_rows && start.v[b] + i < a.capacity, a.err)) dst[row * ru + e] = src[u];
    }
}

cudaError_t launch_cache_append(const Shape& s, const tpa_cache& c, const tpa_factors& kv,
                                int batch, int n_tokens, const SeqParams& start, int* err,
                                cudaStream_t st) {
    const int es = s.bf16 ? 2 : 4;
    const int n_arr = s.shared ? 2 : 4;       // shared basis: A_K, A_V only
    long long row_bytes[4] = {(long long)s.H * s.Rk * es, (long long)s.H * s.Rv * es,
                              (long long)s.Rk * s.Dh * es, (long long)s.Rv * s.Dh * es};
    // widest vector that divides every row (pointers are 16-byte aligned by contract)
    int vec = 16;
    for (int i = 0; i < n_arr; ++i)
        while (row_bytes[i] % vec) vec >>= 1;
    AppendArgs a;
    a.src[0] = (const char*)kv.a_k; a.src[1] = (const char*)kv.a_v;
    a.src[2] = (const char*)kv.b_k; a.src[3] = (const char*)kv.b_v;
    a.dst[0] = (char*)c.a_k; a.dst[1] = (char*)c.a_v;
    a.dst[2] = (char*)c.b_k; a.dst[3] = (char*)c.b_v;
    for (int i = 0; i < 4; ++i) a.row_units[i] = row_bytes[i] / vec;
    a.batch = batch; a.n_tokens = n_tokens; a.capacity = c.capacity; a.lengths = c.lengths;
    a.dst_rows = (long long)c.batch * c.capacity; a.n_lengths = c.batch; a.err = err;
    long long most = 0;
    for (int i = 0; i < n_arr; ++i) {
        long long t = (long long)batch * n_tokens * a.row_units[i];
        if (t > most) most = t;
    }
    int threads = 256;
    long long blocks = (most + threads - 1) / threads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    dim3 grid((unsigned)blocks, (unsigned)n_arr);
    switch (vec) {
        case 16: append_kernel<uint4><<<grid, threads, 0, st>>>(a, start); break;
        case 8: append_kernel<uint2><<<grid, threads, 0, st>>>(a, start); break;
        case 4: append_kernel<uint32_t><<<grid, threads, 0, st>>>(a, start); break;
        default: append_kernel<uint16_t><<<grid, threads, 0, st>>>(a, start); break;
    }
    return cudaGetLastError();
}

// table_k[p][s][2k, 2k+1] = basis_k[s] pair k turned by cs[p][k] (the rotation and the
// fp32 arithmetic of the projection epilogue's RoPE); table_v[p][s][:] = basis_v[s].
template <typename T>
__global__ void basis_table_kernel(const T* __restrict__ bk, const T* __restrict__ bv,
                                   const float2* __restrict__ cs, int capacity, int Rk, int Rv,
                                   int half, T* __restrict__ tk, T* __restrict__ tv) {
    const long long step = (long long)gridDim.x * blockDim.x;
    const long long t0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const int d = 2 * half;
    const long long nk = (long long)capacity * Rk * half;
    for (long long u = t0; u < nk; u += step) {
        const int k = (int)(u % half);
        const long long ps = u / half;             // p * Rk + s
        const int sr = (int)(ps % Rk);
        const int p = (int)(ps / Rk);
        const float x0 = to_f(bk[(long long)sr * d + 2 * k]);
        const float x1 = to_f(bk[(long long)sr * d + 2 * k + 1]);
        const float2 r = cs[(long long)p * half + k];
        tk[ps * d + 2 * k] = from_f<T>(x0 * r.x - x1 * r.y);
        tk[ps * d + 2 * k + 1] = from_f<T>(x0 * r.y + x1 * r.x);
    }
    const long long nv = (long long)capacity * Rv * d;
    const long long per = (long long)Rv * d;
    for (long long u = t0; u < nv; u += step) tv[u] = bv[u % per];
}

cudaError_t launch_shared_basis_tables(const Shape& s, const void* basis_k, const void* basis_v,
                                       const float* cs, int capacity, void* table_k,
                                       void* table_v, cudaStream_t st) {
    const long long work = (long long)capacity * (s.Rk * s.Dh / 2 + s.Rv * s.Dh);
    long long blocks = (work + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    const float2* c2 = reinterpret_cast<const float2*>(cs);
    if (s.bf16)
        basis_table_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(basis_k), static_cast<const __nv_bfloat16*>(basis_v), c2,
            capacity, s.Rk, s.Rv, s.Dh / 2, static_cast<__nv_bfloat16*>(table_k),
            static_cast<__nv_bfloat16*>(table_v));
    else
        basis_table_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
            static_cast<const float*>(basis_k), static_cast<const float*>(basis_v), c2, capacity,
            s.Rk, s.Rv, s.Dh / 2, static_cast<float*>(table_k), static_cast<float*>(table_v));
    return cudaGetLastError();
}

}  // namespace tpa
