// Internal interface between the C ABI (tpa_api.cu) and the kernels.  Not installed.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/tpa.h"

namespace tpa {

// Per-sequence host values (start positions or lengths), passed by value as a kernel
// parameter so that no device copy (and no allocation) is needed.
struct SeqParams {
    int32_t v[TPA_MAX_BATCH];
};

struct Shape {
    int D, H, Dh, Rq, Rk, Rv;
    bool bf16;
    bool shared;    // shared basis: B_K, B_V are per-position tables, one for all sequences
};

inline Shape shape_of(const tpa_dims& d) {
    return Shape{d.d_model, d.n_heads, d.head_dim, d.rank_q, d.rank_k, d.rank_v,
                 d.dtype == TPA_BF16, d.shared_basis != 0};
}

// Cache rows between sequences in the B_K / B_V tensors: the capacity, or 0 for a
// shared basis (every sequence reads the same per-position table).
inline long long b_seq_rows(const Shape& s, const tpa_cache& c) {
    return s.shared ? 0 : (long long)c.capacity;
}

// Column layout of the stacked projection output: [a_q | a_k | a_v | b_q | b_k | b_v].
// TPA-KVonly (rank_q = 0): a_q is empty and the b_q segment is the plain query
// projection, h rows of d_h ([T][h][d_h]), rotated like B_Q.  Shared basis: the b_k
// and b_v segments are empty (no column maps to them).
struct ProjLayout {
    int off[7];    // segment starts, off[6] = N
    void* dst[6];  // a_q, a_k, a_v, b_q, b_k, b_v
    // Cache mode (kv_cap > 0): dst[1,2,4,5] are the cache's a_k, a_v, b_k, b_v and
    // token t = b*seqlen + i lands in cache row b*kv_cap + start[b] + i; the kernel
    // also sets lengths[b] = start[b] + seqlen.  Otherwise every segment is at row t.
    int kv_cap = 0;
    int32_t* lengths = nullptr;
    // Extents for the bounds-checked build: destination rows of each segment, entries
    // of `lengths`, rows of the RoPE table.
    long long rows[6] = {0, 0, 0, 0, 0, 0};
    int n_lengths = 0;
    int cs_rows = 0;
};

// Destination row of segment s for token t (tkv: its cache row in cache mode).
__host__ __device__ inline long long seg_row(const ProjLayout& L, int s, long long t, long long tkv) {
    return (L.kv_cap > 0 && s != 0 && s != 3) ? tkv : t;
}

inline ProjLayout proj_layout(const Shape& s, const tpa_factors& f, long long T, int cs_rows) {
    ProjLayout L;
    for (int i = 0; i < 6; ++i) L.rows[i] = T;
    L.cs_rows = cs_rows;
    const int q_rows = s.Rq > 0 ? s.Rq : s.H;
    int w[6] = {s.H * s.Rq, s.H * s.Rk, s.H * s.Rv, q_rows * s.Dh,
                s.shared ? 0 : s.Rk * s.Dh, s.shared ? 0 : s.Rv * s.Dh};
    L.off[0] = 0;
    for (int i = 0; i < 6; ++i) L.off[i + 1] = L.off[i] + w[i];
    L.dst[0] = f.a_q; L.dst[1] = f.a_k; L.dst[2] = f.a_v;
    L.dst[3] = f.b_q; L.dst[4] = f.b_k; L.dst[5] = f.b_v;
    return L;
}

// Decode plan.  Each sequence's context is cut into pieces ("parts"); every part
// leaves one partial softmax state (m, l, o) per head in the workspace, and the
// combine kernel merges the parts of a sequence in part order.  The parts of
// sequence b are first_part[b] .. first_part[b] + n_parts[b] - 1.
//  - CUDA-core decode: parts are splits of split_len keys; CTA (split, b).
//  - tensor-core decode: a persistent grid of n_ctas CTAs walks the concatenated
//    key tiles of all sequences; CTA c takes tiles [c*N/G, (c+1)*N/G), and each
//    (CTA, sequence) overlap is one part; c_first[b] is the first CTA on sequence b.
//  - paired (shared-basis decode at h 16): the walk is over units of two sequences
//    (2u, 2u+1) that share each key tile; tile_prefix and c_first are per unit, and
//    a unit's CTAs give each member its own consecutive parts.
struct DecodePlan {
    int32_t len[TPA_MAX_BATCH];
    int32_t first_part[TPA_MAX_BATCH];
    int32_t n_parts[TPA_MAX_BATCH];
    int32_t tile_prefix[TPA_MAX_BATCH + 1];
    int32_t c_first[TPA_MAX_BATCH];
    int32_t batch, n_ctas, total_tiles, total_parts, split_len, key_tile;
    int32_t pairs;       // units of two sequences (paired plan)
    int32_t n_units;     // units walked: batch, or ceil(batch / 2) when paired
};

// The shared-basis decode at h 16 pairs sequences (tensor-core path only).
inline bool decode_pairs(const Shape& s) { return s.shared && s.H == 16; }

// Builds the plan for the decode kernel that handles this shape (tc = tensor-core path).
void make_decode_plan(const Shape& s, const int32_t* lengths, int batch, bool tc,
                      DecodePlan* plan);
size_t decode_workspace_bytes(const Shape& s, const DecodePlan& plan);

// Every check tpa_decode makes before it looks at the workspace: dims, cache, query,
// output and lengths.  tpa_decode_static shares it, so both return the same status.
tpa_status validate_decode(const tpa_dims* d, const void* q_a, const void* q_b,
                           const tpa_cache* c, const int32_t* lengths, int32_t batch,
                           const void* out);

// ---- launchers (each returns the launch's cudaError_t) ----
cudaError_t launch_rope_table(float* cs, int max_pos, int head_dim, double base,
                              cudaStream_t st);

cudaError_t launch_project_simt(const Shape& s, const void* x, const void* w, int batch,
                                int seqlen, const SeqParams& start, const float* cs,
                                const ProjLayout& L, int* err, cudaStream_t st);

cudaError_t launch_project_tc(const Shape& s, const void* x, const void* w, int batch,
                              int seqlen, const SeqParams& start, const float* cs,
                              const ProjLayout& L, int* err, uint32_t wait_limit,
                              cudaStream_t st);
bool project_tc_supported(const Shape& s, int T);

cudaError_t launch_shared_basis_tables(const Shape& s, const void* basis_k, const void* basis_v,
                                       const float* cs, int capacity, void* table_k,
                                       void* table_v, cudaStream_t st);

cudaError_t launch_cache_append(const Shape& s, const tpa_cache& c, const tpa_factors& kv,
                                int batch, int n_tokens, const SeqParams& start, int* err,
                                cudaStream_t st);

cudaError_t launch_prefill_simt(const Shape& s, const tpa_factors& q, const tpa_cache& c,
                                int batch, int seqlen, const SeqParams& start, void* out,
                                int* err, cudaStream_t st);

cudaError_t launch_prefill_tc(const Shape& s, const tpa_factors& q, const tpa_cache& c,
                              int batch, int seqlen, const SeqParams& start, void* out,
                              int* err, uint32_t wait_limit, cudaStream_t st);
bool prefill_tc_supported(const Shape& s);

// Query-major prefill (K and V formed per tile in shared memory); preferred where supported.
cudaError_t launch_prefill_qm(const Shape& s, const tpa_factors& q, const tpa_cache& c,
                              int batch, int seqlen, const SeqParams& start, void* out,
                              int* err, uint32_t wait_limit, cudaStream_t st);
bool prefill_qm_supported(const Shape& s);

cudaError_t launch_decode_simt(const Shape& s, const void* q_a, const void* q_b,
                               const tpa_cache& c, const DecodePlan& plan, float* ws, int* err,
                               cudaStream_t st);

cudaError_t launch_decode_tc(const Shape& s, const void* q_a, const void* q_b,
                             const tpa_cache& c, const DecodePlan& plan, float* ws, int* err,
                             uint32_t wait_limit, cudaStream_t st);
bool decode_tc_supported(const Shape& s);

cudaError_t launch_decode_combine(const Shape& s, const DecodePlan& plan, const float* ws,
                                  void* out, int* err, cudaStream_t st);

}  // namespace tpa
