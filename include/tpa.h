/*
 * tpa.h - C ABI of libtpa.so: the data-parallel hot path of Tensor Product Attention
 * (TPA) on NVIDIA B200 (sm_100a).
 *
 * TPA writes each token's query, key and value as a contextual rank-R sum
 *     Q_t = (1/R_Q) sum_r a_r^Q(x_t) (outer) b_r^Q(x_t),  a_r in R^h, b_r in R^{d_h}
 * and likewise for K (R_K) and V (R_V)  ["【拜读】Tensor Product Attention Is All You Need
 * 姚期智团队开源兼容RoPE位置编码" (coreui.cn), 核心机制总结 §3 公式描述].  Only the factors
 * are cached, B_K already rotated by RoPE at its position [same page, 关键问题及回答 问题2],
 * and attention softmax(Q K^T / sqrt(d_h)) V ["张量积注意力（TPA）…" (jieyibu.net), Ⅱ.1]
 * is computed from the cached factors; K and V are never written to device memory.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers marked "device" point to device memory of the current CUDA device;
 *    pointers marked "host" point to host memory read before the call returns.
 *    The caller owns every buffer; the library allocates nothing and keeps no
 *    pointer after the call returns.  Its only global state is one 32-bit device
 *    error word per device (tpa_get_device_error) and the fixed scratch array of
 *    tpa_decode_static, both file-scope device variables of the library.
 *  - Every compute call is asynchronous on `stream` (a cudaStream_t; NULL means the
 *    legacy default stream).  Arguments are validated on the host before any launch;
 *    a call that returns an error has launched nothing.  TPA_ERR_CUDA means a launch
 *    failed; the CUDA error is left for cudaGetLastError().
 *  - Element type: dims->dtype selects fp32 (TPA_F32) or bf16 (TPA_BF16) for every
 *    factor, cache, query and output buffer of the call; x and w_cat use it too.
 *    Arithmetic is fp32 (bf16 operands on tensor cores, fp32 accumulation and softmax).
 *  - Layouts are dense row-major with the shapes given below, T = batch * seqlen tokens
 *    ordered sequence-major (token t = b * seqlen + i).  The A and B factor layouts
 *    follow the page's views: A_* is [.., h, R] (head-major) and B_* is [.., R, d_h]
 *    [review, 代码 前向传播].  Device pointers must be 16-byte aligned.
 *  - Factors are stored raw, without the 1/R; attention applies 1/R_Q, 1/R_K, 1/R_V
 *    and 1/sqrt(d_h).  B_Q and B_K leave tpa_project already rotated.
 *  - RoPE: interleaved pairs (2k, 2k+1) of the head dimension turn by p * theta_k,
 *    theta_k = base^(-2k/d_h), p the 0-based absolute position (the LLaMA convention
 *    behind the page's freqs_cis / apply_rotary_emb, whose body the pages do not print).
 *  - Kernels never trap.  Where a kernel waits on a barrier it gives up after a bounded
 *    number of tries, records TPA_DEVERR_TIMEOUT in the device error word and returns.
 *    The outputs of a call for which tpa_get_device_error then reports an error are
 *    undefined.
 *  - The library looks up the device address of its error word (and of the
 *    tpa_decode_static scratch array) once per device and keeps it; it must not be
 *    used across cudaDeviceReset or any other re-creation of a device's context.
 */
#ifndef TPA_H
#define TPA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TPA_ABI_VERSION 2
#define TPA_MAX_BATCH 1024          /* sequences per call */

typedef struct CUstream_st* tpa_stream_t;   /* same type as cudaStream_t */

typedef enum tpa_status {
    TPA_OK = 0,
    TPA_ERR_INVALID = 1,        /* null pointer, bad size, misaligned pointer, bad position */
    TPA_ERR_UNSUPPORTED = 2,    /* valid TPA shape that no kernel here implements */
    TPA_ERR_CAPACITY = 3,       /* write past the cache capacity or the RoPE table */
    TPA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
    TPA_ERR_WORKSPACE = 5,      /* workspace too small */
    TPA_ERR_DEVICE = 6          /* tpa_get_device_error found a recorded device error */
} tpa_status;

typedef enum tpa_dtype { TPA_F32 = 0, TPA_BF16 = 1 } tpa_dtype;

/* device error word values (tpa_get_device_error) */
#define TPA_DEVERR_NONE 0
#define TPA_DEVERR_TIMEOUT 1        /* a bounded wait gave up */
#define TPA_DEVERR_BOUNDS 2         /* an index check failed (debug builds) */

/* Shape of one TPA layer: the page's ModelArgs (dim, n_heads, head_dim, q_rank, rank)
 * [review, 代码 类定义与初始化], with rank split into rank_k and rank_v.
 * rank_q = 0 selects TPA-KVonly [review, 实验/结果]: the query is a plain per-head
 * vector [h][d_h] held in the b_q slot; a_q is unused.
 * shared_basis = 1 selects the variant that shares the basis vectors across tokens
 * [review, 优点与创新 5], named there in one clause.  Reading taken: B_K and B_V are
 * layer parameters (basis_k [R_K][d_h], basis_v [R_V][d_h]), the same for every
 * token; A_K, A_V and the query stay contextual; RoPE turns the key at its position.
 * Only A_K and A_V are cached per token.  The per-call effects are stated below. */
typedef struct tpa_dims {
    int32_t d_model;
    int32_t n_heads;     /* h */
    int32_t head_dim;    /* d_h, even */
    int32_t rank_q;      /* R_Q (0: KV-only) */
    int32_t rank_k;      /* R_K */
    int32_t rank_v;      /* R_V */
    int32_t dtype;       /* tpa_dtype */
    int32_t shared_basis;  /* 0: contextual B_K, B_V (TPA); 1: shared basis */
} tpa_dims;

/* The six factor tensors of T tokens (device):
 *   a_q [T][h][R_Q]   a_k [T][h][R_K]   a_v [T][h][R_V]
 *   b_q [T][R_Q][d_h] b_k [T][R_K][d_h] b_v [T][R_V][d_h]   (b_q, b_k rotated)
 * TPA-KVonly (rank_q = 0): b_q holds the rotated query [T][h][d_h]; a_q may be NULL. */
typedef struct tpa_factors {
    void* a_q; void* b_q;
    void* a_k; void* b_k;
    void* a_v; void* b_v;
} tpa_factors;

/* The factor cache of `batch` sequences with room for `capacity` tokens each (device),
 * the page's cache_kA / cache_vA / cache_kB / cache_vB [review, 类定义与初始化]:
 *   a_k, a_v [batch][capacity][h][R]    b_k, b_v [batch][capacity][R][d_h]
 * lengths [batch] int32 (device) is written by tpa_cache_append.
 * Shared basis (dims->shared_basis = 1): b_k and b_v are the layer's per-position
 * tables [capacity][R][d_h] from tpa_shared_basis_tables, read by every sequence. */
typedef struct tpa_cache {
    void* a_k; void* a_v;
    void* b_k; void* b_v;
    int32_t* lengths;
    int32_t batch;
    int32_t capacity;
} tpa_cache;

/* ABI version (TPA_ABI_VERSION) and a short description of the library build. */
int32_t tpa_abi_version(void);
const char* tpa_build_info(void);
const char* tpa_status_string(tpa_status status);

/* Bytes the factor cache holds per token: (R_K + R_V) * (h + d_h) * sizeof(element),
 * from the page's cache shapes [review, 类定义与初始化]; (R_K + R_V) * h * sizeof(element)
 * with a shared basis (the per-layer tables are not per token).  0 for invalid dims. */
size_t tpa_cache_bytes_per_token(const tpa_dims* dims);

/* RoPE table: cs[p][k][0] = cos(p * theta_k), cs[p][k][1] = sin(p * theta_k) for
 * p < max_pos, k < d_h/2, angles formed and evaluated in fp64, stored as fp32.
 * cs: device float [max_pos][d_h/2][2].  This is the caller-supplied freqs_cis of
 * the page's forward(x, start_pos, freqs_cis, mask) [review, 代码 前向传播]. */
tpa_status tpa_rope_table(const tpa_dims* dims, double base, int32_t max_pos,
                          float* cs, tpa_stream_t stream);

/* Factor projection: Y = x W_cat^T, cut into the six factors, with RoPE applied to
 * the B_Q and B_K columns of token t = b*seqlen+i at position start_pos[b] + i.
 * The six bias-free projections W_A_q/k/v, W_B_q/k/v of [review, 类定义与初始化 /
 * 前向传播], fused into one GEMM; RoPE on B before caching per [review, 问题2].
 *   x      device [T][d_model]
 *   w_cat  device [N][d_model], N = h(R_Q+R_K+R_V) + d_h(R_Q+R_K+R_V): the six
 *          nn.Linear weights stacked in the order W_A_q, W_A_k, W_A_v, W_B_q, W_B_k, W_B_v
 *   start_pos host [batch]; every start_pos[b] + seqlen <= max_pos (else TPA_ERR_CAPACITY)
 *   rope_cs device table from tpa_rope_table with the same head_dim and >= max_pos rows
 *   out    device factor buffers for T tokens (all six set, none aliasing x or w_cat)
 * TPA-KVonly (rank_q = 0): the W_A_q block is empty and the W_B_q block is the plain
 * query projection W_Q with h*d_h rows (row h*d_h + k is head h, dim k), so N =
 * h(R_K+R_V) + d_h(h+R_K+R_V); out->b_q receives the rotated query [T][h][d_h] and
 * out->a_q may be NULL.  The pages do not print this variant's projection; this
 * layout is the reading taken.
 * Shared basis: the W_B_k and W_B_v blocks are absent (N = h(R_Q+R_K+R_V) + d_h R_Q,
 * or the KV-only count without them) and out->b_k, out->b_v are not used (may be NULL). */
tpa_status tpa_project(const tpa_dims* dims, const void* x, const void* w_cat,
                       int32_t batch, int32_t seqlen, const int32_t* start_pos,
                       const float* rope_cs, int32_t max_pos,
                       const tpa_factors* out, tpa_stream_t stream);

/* Cache append: for every sequence b and i < n_tokens, copy token b*n_tokens+i of
 * kv->a_k, kv->a_v, kv->b_k, kv->b_v into cache position start_pos[b] + i, bit for
 * bit, and set cache->lengths[b] = start_pos[b] + n_tokens.  The page's
 * cache[:bsz, start_pos:start_pos+seqlen] = factors [review, 代码 前向传播].
 *   kv         device factors for batch*n_tokens tokens (a_q, b_q ignored)
 *   start_pos  host [batch]; start_pos[b] + n_tokens <= capacity (else TPA_ERR_CAPACITY)
 * batch <= cache->batch; sequences >= batch are left alone.
 * Shared basis: only a_k and a_v are copied; kv->b_k, kv->b_v may be NULL. */
tpa_status tpa_cache_append(const tpa_dims* dims, const tpa_cache* cache,
                            const tpa_factors* kv, int32_t batch, int32_t n_tokens,
                            const int32_t* start_pos, tpa_stream_t stream);

/* Shared-basis tables (dims->shared_basis = 1) for a cache of `capacity` positions:
 *   table_k[p][s][:] = basis_k[s] rotated at position p (RoPE as tpa_project rotates
 *                      B_K: fp32 arithmetic, rounded once to dims->dtype)
 *   table_v[p][s][:] = basis_v[s]
 * This is the cache side of the shared basis, pre-rotated as B_K is cached [review,
 * 问题2]: one table per layer, not per sequence.  Set cache->b_k = table_k and
 * cache->b_v = table_v.  Rebuild after changing the basis.
 *   basis_k  device [R_K][d_h]      basis_v device [R_V][d_h]
 *   rope_cs  device table from tpa_rope_table with max_pos >= capacity rows
 *   table_k  device [capacity][R_K][d_h]   table_v device [capacity][R_V][d_h]
 * TPA_ERR_INVALID if dims->shared_basis is 0; TPA_ERR_CAPACITY if capacity > max_pos. */
tpa_status tpa_shared_basis_tables(const tpa_dims* dims, const void* basis_k,
                                   const void* basis_v, const float* rope_cs,
                                   int32_t max_pos, int32_t capacity, void* table_k,
                                   void* table_v, tpa_stream_t stream);

/* Causal prefill from factors: query i of sequence b (position p = start_pos[b] + i)
 * attends to cached keys 0..p of sequence b:
 *   out[b*seqlen+i][h][:] = sum_j softmax_j(q_h . k_{j,h} / sqrt(d_h)) v_{j,h}
 * with q, k, v the (1/R) rank sums of the factors [review, §3 公式描述 and 前向传播;
 * jieyibu.net page, Ⅱ.1], evaluated from the factors without writing K or V out.
 *   q      device a_q, b_q (rotated) for batch*seqlen tokens (other members ignored);
 *          TPA-KVonly: b_q = the rotated query [T][h][d_h], a_q ignored
 *   cache  must already hold positions 0 .. start_pos[b]+seqlen-1 of each sequence
 *   start_pos host [batch]
 *   out    device [batch*seqlen][h][d_h]
 * Shared basis: key j of every sequence reads row j of cache->b_k and cache->b_v. */
tpa_status tpa_prefill(const tpa_dims* dims, const tpa_factors* q, const tpa_cache* cache,
                       int32_t batch, int32_t seqlen, const int32_t* start_pos,
                       void* out, tpa_stream_t stream);

/* Decode: one query per sequence at position lengths[b]-1 attends to cached keys
 * 0..lengths[b]-1 (the new token is appended first: the page writes the cache before
 * reading it [review, 代码 前向传播]).  Keys are read only as factors, B_K used as cached
 * (pre-rotated, so decode rotates nothing [review, 问题2]).  The context is split
 * across CTAs and the partial softmax states are merged in a fixed order, so results
 * are run-to-run identical.
 *   q_a      device [batch][h][R_Q] (NULL when rank_q == 0)
 *   q_b      device [batch][R_Q][d_h] rotated at lengths[b]-1, or the rotated per-head
 *            query [batch][h][d_h] when rank_q == 0 (TPA-KVonly)
 *   lengths  host [batch], 1 <= lengths[b] <= capacity
 *   out      device [batch][h][d_h]
 *   workspace device scratch of at least tpa_decode_workspace_bytes() bytes, 256-byte
 *            aligned; contents on entry do not matter and are undefined on return.
 * Shared basis: keys read A_K, A_V from the sequence's cache rows and B_K, B_V from
 * the per-position tables (so per key only (R_K + R_V) h elements come from HBM). */
tpa_status tpa_decode(const tpa_dims* dims, const void* q_a, const void* q_b,
                      const tpa_cache* cache, const int32_t* lengths, int32_t batch,
                      void* out, void* workspace, size_t workspace_bytes,
                      tpa_stream_t stream);

/* Workspace bytes tpa_decode needs for these lengths (0 for invalid arguments). */
size_t tpa_decode_workspace_bytes(const tpa_dims* dims, const int32_t* lengths, int32_t batch);

/* One decode step from the hidden state of the new token of every sequence: project
 * it (the six projections with RoPE at position lengths[b], as tpa_project), write
 * its A_K, A_V, B_K, B_V into the cache at position lengths[b] and set
 * cache->lengths[b] = lengths[b] + 1 (as tpa_cache_append), then decode its query
 * over keys 0..lengths[b] (as tpa_decode).  This is the page's forward for one token
 * with start_pos = lengths[b]: project, write the cache, read it back, attend
 * [review, 代码 前向传播].  Two stream-ordered kernel launches plus decode's merge:
 * the projection's epilogue writes the key/value factors straight into the cache,
 * so they never pass through a separate buffer.
 *   x        device [batch][d_model]: the new token of each sequence
 *   w_cat    device stacked weights, as tpa_project (TPA-KVonly layout at rank_q = 0)
 *   rope_cs  device table from tpa_rope_table with max_pos rows; lengths[b] < max_pos
 *   cache    holds positions 0 .. lengths[b]-1 of sequence b; lengths[b] + 1 <= capacity
 *   lengths  host [batch], lengths[b] >= 0: the cached length before this step
 *   out      device [batch][h][d_h]
 *   workspace device scratch of at least tpa_decode_step_workspace_bytes() bytes,
 *            256-byte aligned: the new tokens' query factors, then decode's partials.
 * Arguments are checked before anything is launched (TPA_ERR_CAPACITY when a
 * sequence has no room or its position is past the RoPE table).
 * Shared basis: only A_K, A_V are written into the cache (w_cat without W_B_k, W_B_v). */
tpa_status tpa_decode_step(const tpa_dims* dims, const void* x, const void* w_cat,
                           const float* rope_cs, int32_t max_pos, const tpa_cache* cache,
                           const int32_t* lengths, int32_t batch, void* out,
                           void* workspace, size_t workspace_bytes, tpa_stream_t stream);

/* Output projection: out = attn W_o^T, the layer's closing self.wo(output) [review, 代码
 * 前向传播], with the attention output flattened head-major per token (feature
 * h*d_h + k is head h, dim k, as transpose(1,2).view(bsz, seqlen, -1)).  The page
 * uses wo without defining it; reading taken: a bias-free nn.Linear(h*d_h, d_model).
 * The T6GroupNorm the page constructs is not applied in its forward and is not here.
 *   attn  device [T][h][d_h] (tpa_prefill's or tpa_decode's out)
 *   w_o   device [d_model][h*d_h]
 *   out   device [T][d_model]
 * Same element type throughout (dims->dtype); fp32 accumulation. */
tpa_status tpa_output_project(const tpa_dims* dims, const void* attn, const void* w_o,
                              int32_t T, void* out, tpa_stream_t stream);

/* Workspace bytes tpa_decode_step needs for these pre-step lengths (0 if invalid). */
size_t tpa_decode_step_workspace_bytes(const tpa_dims* dims, const int32_t* lengths,
                                       int32_t batch);

/* tpa_decode without a caller-supplied workspace, for callers that cannot allocate
 * device memory: a host application that owns every allocation and hands this
 * library only its inputs and outputs, or a server that must not call cudaMalloc
 * once it is running.  The paper has no counterpart; this is a deployment variant.
 * The split-K scratch is a file-scope device array of TPA_DECODE_STATIC_SCRATCH_BYTES
 * that every GPU loading the library holds until the process exits.  The first call
 * on each device looks up that array's address (make it before any stream capture).
 * The cached address is only valid in the context it was looked up in: do not use
 * the library across cudaDeviceReset (or any re-creation of the device's primary
 * context).  Arguments are checked as tpa_decode checks them, with the same status
 * codes; then calls needing more scratch than the array holds (see
 * tpa_decode_workspace_bytes) return TPA_ERR_WORKSPACE.  Both checks come before any
 * CUDA call.  All calls on a device share the array, so calls that overlap on the
 * GPU race: keep them ordered on one stream.  Nothing needs clearing between calls;
 * but when tpa_get_device_error reports an error for a call, that call's output is
 * undefined (it may mix in partial states an earlier call left in the array).
 * Allocates nothing.  Arguments and results are otherwise those of tpa_decode. */
#define TPA_DECODE_STATIC_SCRATCH_BYTES (16u << 20)
tpa_status tpa_decode_static(const tpa_dims* dims, const void* q_a, const void* q_b,
                             const tpa_cache* cache, const int32_t* lengths, int32_t batch,
                             void* out, tpa_stream_t stream);

/* Which kernel family a call with these dims runs (host query, no CUDA call):
 *   TPA_FAMILY_TENSOR_CORE  the tcgen05 / TMA kernels (bf16 shapes they cover)
 *   TPA_FAMILY_CUDA_CORE    the CUDA-core kernels (fp32, and bf16 shapes outside the
 *                           tensor-core kernels' limits: see each kernel's limits)
 *   TPA_FAMILY_NONE         the dims are invalid or the call is unsupported for them
 * call: TPA_CALL_PROJECT (tpa_project, tpa_output_project and the projection half of
 * tpa_decode_step), TPA_CALL_PREFILL, TPA_CALL_DECODE (tpa_decode, tpa_decode_static
 * and the decode half of tpa_decode_step).  Lets a caller or a benchmark assert that
 * its shape takes the tensor-core path rather than learn it from a profiler. */
#define TPA_CALL_PROJECT 0
#define TPA_CALL_PREFILL 1
#define TPA_CALL_DECODE 2
#define TPA_FAMILY_NONE (-1)
#define TPA_FAMILY_CUDA_CORE 0
#define TPA_FAMILY_TENSOR_CORE 1
int32_t tpa_kernel_family(const tpa_dims* dims, int32_t call);

/* Synchronise `stream`, then read and clear the device error word of the current
 * device.  *code receives the TPA_DEVERR_* value (NULL allowed).  Returns TPA_OK if
 * it was clear, TPA_ERR_DEVICE if a kernel recorded an error, TPA_ERR_CUDA if the
 * synchronisation itself failed. */
tpa_status tpa_get_device_error(tpa_stream_t stream, int32_t* code);

/* Test hook: the number of polls a bounded wait makes before it gives up
 * (0 restores the default).  Host-side setting, read at each launch. */
void tpa_set_wait_limit(uint32_t polls);

#ifdef __cplusplus
}
#endif
#endif /* TPA_H */
