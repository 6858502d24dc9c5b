// The C ABI of libtpa.so (declared in include/tpa.h): host-side validation, the
// per-device error word, and dispatch to the kernels.  No call allocates memory.
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "tpa_internal.h"

namespace tpa {
// One error word per device; kernels record the first failure here (never trap).
__device__ int g_device_error;
}  // namespace tpa

using namespace tpa;

namespace {

std::atomic<uint32_t> g_wait_limit{0};
constexpr uint32_t kDefaultWaitLimit = 1u << 24;   // polls: at most seconds of waiting
constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
int* g_err_ptr[kMaxDevices] = {};

uint32_t wait_limit() {
    uint32_t v = g_wait_limit.load(std::memory_order_relaxed);
    return v ? v : kDefaultWaitLimit;
}

// Device address of the error word on the current device (looked up once per device).
int* device_error_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_err_mu);
    if (!g_err_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<int*>(p);
    }
    return g_err_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks common to all calls.  need_q: the call reads factorised queries.
tpa_status check_dims(const tpa_dims* d, bool need_q) {
    if (!d) return TPA_ERR_INVALID;
    if (d->dtype != TPA_F32 && d->dtype != TPA_BF16) return TPA_ERR_INVALID;
    if (d->n_heads < 1 || d->head_dim < 2 || (d->head_dim & 1)) return TPA_ERR_INVALID;
    if (d->rank_k < 1 || d->rank_v < 1 || d->rank_q < 0) return TPA_ERR_INVALID;
    if (d->shared_basis != 0 && d->shared_basis != 1) return TPA_ERR_INVALID;
    if (need_q && d->rank_q < 1) return TPA_ERR_UNSUPPORTED;
    if (d->n_heads > 4096 || d->head_dim > 4096 || d->rank_q > 256 || d->rank_k > 256 ||
        d->rank_v > 256)
        return TPA_ERR_UNSUPPORTED;
    return TPA_OK;
}

tpa_status check_cache(const tpa_cache* c, int batch) {
    if (!c || !c->a_k || !c->a_v || !c->b_k || !c->b_v || !c->lengths) return TPA_ERR_INVALID;
    if (!aligned16(c->a_k) || !aligned16(c->a_v) || !aligned16(c->b_k) || !aligned16(c->b_v))
        return TPA_ERR_INVALID;
    if (c->capacity < 1 || c->batch < 1 || batch < 1 || batch > c->batch ||
        batch > TPA_MAX_BATCH)
        return TPA_ERR_INVALID;
    return TPA_OK;
}

tpa_status launched(cudaError_t e) { return e == cudaSuccess ? TPA_OK : TPA_ERR_CUDA; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace bytes tpa_decode_step keeps for the new tokens' query factors (a_q, then
// b_q or the KV-only query), each 256-byte aligned.
size_t step_query_bytes(const Shape& s, int batch) {
    const size_t es = s.bf16 ? 2 : 4;
    const size_t q_rows = s.Rq > 0 ? (size_t)s.Rq : (size_t)s.H;
    return round_up((size_t)batch * s.H * s.Rq * es, 256) + round_up((size_t)batch * q_rows * s.Dh * es, 256);
}

// The projection GEMM with its fused epilogue (validated arguments).
tpa_status run_project(const Shape& s, const void* x, const void* w, int batch, int seqlen,
                       const SeqParams& sp, const float* rope_cs, const ProjLayout& L,
                       cudaStream_t cs) {
    if (s.bf16 && project_tc_supported(s, batch * seqlen))
        return launched(launch_project_tc(s, x, w, batch, seqlen, sp, rope_cs, L,
                                          device_error_ptr(), wait_limit(), cs));
    return launched(launch_project_simt(s, x, w, batch, seqlen, sp, rope_cs, L, device_error_ptr(), cs));
}

// Split-K decode and the fixed-order merge of its parts (validated arguments).
tpa_status run_decode(const Shape& s, const void* q_a, const void* q_b, const tpa_cache& c,
                      const int32_t* lengths, int batch, void* out, void* workspace,
                      size_t workspace_bytes, cudaStream_t cs) {
    const bool tc = s.bf16 && decode_tc_supported(s);
    if (!tc && (long long)s.H * s.Dh > 8192) return TPA_ERR_UNSUPPORTED;
    DecodePlan plan;
    make_decode_plan(s, lengths, batch, tc, &plan);
    if (decode_workspace_bytes(s, plan) > workspace_bytes) return TPA_ERR_WORKSPACE;
    float* ws = static_cast<float*>(workspace);
    cudaError_t e = tc ? launch_decode_tc(s, q_a, q_b, c, plan, ws, device_error_ptr(), wait_limit(), cs)
                       : launch_decode_simt(s, q_a, q_b, c, plan, ws, device_error_ptr(), cs);
    if (e != cudaSuccess) return TPA_ERR_CUDA;
    return launched(launch_decode_combine(s, plan, ws, out, device_error_ptr(), cs));
}

}  // namespace

namespace tpa {
tpa_status validate_decode(const tpa_dims* d, const void* q_a, const void* q_b,
                           const tpa_cache* c, const int32_t* lengths, int32_t batch,
                           const void* out) {
    tpa_status st = check_dims(d, false);
    if (st != TPA_OK) return st;
    if ((st = check_cache(c, batch)) != TPA_OK) return st;
    if (!q_b || !lengths || !out) return TPA_ERR_INVALID;
    if (d->rank_q > 0 && (!q_a || !aligned16(q_a))) return TPA_ERR_INVALID;
    if (!aligned16(q_b) || !aligned16(out)) return TPA_ERR_INVALID;
    for (int b = 0; b < batch; ++b) {
        if (lengths[b] < 1) return TPA_ERR_INVALID;
        if (lengths[b] > c->capacity) return TPA_ERR_CAPACITY;
    }
    return TPA_OK;
}
}  // namespace tpa

extern "C" {

int32_t tpa_abi_version(void) { return TPA_ABI_VERSION; }

const char* tpa_build_info(void) {
#ifdef TPA_DEBUG_BOUNDS
    return "libtpa: TPA hot path for sm_100a (tcgen05/TMA kernels for bf16, CUDA-core "
           "kernels for fp32), bounds-checked build";
#else
    return "libtpa: TPA hot path for sm_100a (tcgen05/TMA kernels for bf16, CUDA-core "
           "kernels for fp32)";
#endif
}

const char* tpa_status_string(tpa_status s) {
    switch (s) {
        case TPA_OK: return "ok";
        case TPA_ERR_INVALID: return "invalid argument";
        case TPA_ERR_UNSUPPORTED: return "unsupported shape";
        case TPA_ERR_CAPACITY: return "position beyond cache capacity or RoPE table";
        case TPA_ERR_CUDA: return "CUDA error";
        case TPA_ERR_WORKSPACE: return "workspace too small";
        case TPA_ERR_DEVICE: return "device-side error recorded";
    }
    return "unknown status";
}

size_t tpa_cache_bytes_per_token(const tpa_dims* d) {
    if (check_dims(d, false) != TPA_OK) return 0;
    size_t es = d->dtype == TPA_BF16 ? 2 : 4;
    const size_t per_rank = (size_t)d->n_heads + (d->shared_basis ? 0 : (size_t)d->head_dim);
    return (size_t)(d->rank_k + d->rank_v) * per_rank * es;
}

void tpa_set_wait_limit(uint32_t polls) { g_wait_limit.store(polls); }

tpa_status tpa_rope_table(const tpa_dims* d, double base, int32_t max_pos, float* cs,
                          tpa_stream_t stream) {
    tpa_status st = check_dims(d, false);
    if (st != TPA_OK) return st;
    if (!cs || !aligned16(cs) || max_pos < 1 || !(base > 1.0)) return TPA_ERR_INVALID;
    if ((long long)max_pos * d->head_dim > (1LL << 34)) return TPA_ERR_UNSUPPORTED;
    return launched(launch_rope_table(cs, max_pos, d->head_dim, base, (cudaStream_t)stream));
}

tpa_status tpa_project(const tpa_dims* d, const void* x, const void* w_cat, int32_t batch,
                       int32_t seqlen, const int32_t* start_pos, const float* rope_cs,
                       int32_t max_pos, const tpa_factors* out, tpa_stream_t stream) {
    tpa_status st = check_dims(d, false);
    if (st != TPA_OK) return st;
    if (d->d_model < 1) return TPA_ERR_INVALID;
    if (!x || !w_cat || !start_pos || !rope_cs || !out) return TPA_ERR_INVALID;
    if ((d->rank_q > 0 && !out->a_q) || !out->b_q || !out->a_k || !out->a_v)
        return TPA_ERR_INVALID;
    if (!d->shared_basis && (!out->b_k || !out->b_v)) return TPA_ERR_INVALID;
    if (!aligned16(x) || !aligned16(w_cat) || !aligned16(rope_cs)) return TPA_ERR_INVALID;
    if (batch < 1 || batch > TPA_MAX_BATCH || seqlen < 1 || max_pos < 1)
        return TPA_ERR_INVALID;
    if ((long long)batch * seqlen > (1LL << 30)) return TPA_ERR_UNSUPPORTED;
    // B_Q / B_K segments must start on an even column so RoPE pairs stay together
    if ((d->n_heads * (d->rank_q + d->rank_k + d->rank_v)) & 1) return TPA_ERR_UNSUPPORTED;
    SeqParams sp;
    for (int b = 0; b < batch; ++b) {
        if (start_pos[b] < 0) return TPA_ERR_INVALID;
        if ((long long)start_pos[b] + seqlen > max_pos) return TPA_ERR_CAPACITY;
        sp.v[b] = start_pos[b];
    }
    Shape s = shape_of(*d);
    return run_project(s, x, w_cat, batch, seqlen, sp, rope_cs,
                       proj_layout(s, *out, (long long)batch * seqlen, max_pos), (cudaStream_t)stream);
}

tpa_status tpa_cache_append(const tpa_dims* d, const tpa_cache* c, const tpa_factors* kv,
                            int32_t batch, int32_t n_tokens, const int32_t* start_pos,
                            tpa_stream_t stream) {
    tpa_status st = check_dims(d, false);
    if (st != TPA_OK) return st;
    if ((st = check_cache(c, batch)) != TPA_OK) return st;
    if (!kv || !kv->a_k || !kv->a_v || !start_pos) return TPA_ERR_INVALID;
    if (!aligned16(kv->a_k) || !aligned16(kv->a_v)) return TPA_ERR_INVALID;
    if (!d->shared_basis &&
        (!kv->b_k || !kv->b_v || !aligned16(kv->b_k) || !aligned16(kv->b_v)))
        return TPA_ERR_INVALID;
    if (n_tokens < 1) return TPA_ERR_INVALID;
    SeqParams sp;
    for (int b = 0; b < batch; ++b) {
        if (start_pos[b] < 0) return TPA_ERR_INVALID;
        if ((long long)start_pos[b] + n_tokens > c->capacity) return TPA_ERR_CAPACITY;
        sp.v[b] = start_pos[b];
    }
    return launched(launch_cache_append(shape_of(*d), *c, *kv, batch, n_tokens, sp,
                                        device_error_ptr(), (cudaStream_t)stream));
}

tpa_status tpa_shared_basis_tables(const tpa_dims* d, const void* basis_k, const void* basis_v,
                                   const float* rope_cs, int32_t max_pos, int32_t capacity,
                                   void* table_k, void* table_v, tpa_stream_t stream) {
    tpa_status st = check_dims(d, false);
    if (st != TPA_OK) return st;
    if (!d->shared_basis) return TPA_ERR_INVALID;
    if (!basis_k || !basis_v || !rope_cs || !table_k || !table_v) return TPA_ERR_INVALID;
    if (!aligned16(basis_k) || !aligned16(basis_v) || !aligned16(rope_cs) ||
        !aligned16(table_k) || !aligned16(table_v))
        return TPA_ERR_INVALID;
    if (capacity < 1 || max_pos < 1) return TPA_ERR_INVALID;
    if (capacity > max_pos) return TPA_ERR_CAPACITY;
    if ((long long)capacity * (d->rank_k + d->rank_v) * d->head_dim > (1LL << 40))
        return TPA_ERR_UNSUPPORTED;
    return launched(launch_shared_basis_tables(shape_of(*d), basis_k, basis_v, rope_cs, capacity,
                                               table_k, table_v, (cudaStream_t)stream));
}

tpa_status tpa_prefill(const tpa_dims* d, const tpa_factors* q, const tpa_cache* c,
                       int32_t batch, int32_t seqlen, const int32_t* start_pos, void* out,
                       tpa_stream_t stream) {
    tpa_status st = check_dims(d, false);
    if (st != TPA_OK) return st;
    if ((st = check_cache(c, batch)) != TPA_OK) return st;
    if (!q || !q->b_q || !start_pos || !out) return TPA_ERR_INVALID;
    if (d->rank_q > 0 && (!q->a_q || !aligned16(q->a_q))) return TPA_ERR_INVALID;
    if (!aligned16(q->b_q) || !aligned16(out)) return TPA_ERR_INVALID;
    if (seqlen < 1) return TPA_ERR_INVALID;
    if (d->head_dim > 256) return TPA_ERR_UNSUPPORTED;
    SeqParams sp;
    for (int b = 0; b < batch; ++b) {
        if (start_pos[b] < 0) return TPA_ERR_INVALID;
        if ((long long)start_pos[b] + seqlen > c->capacity) return TPA_ERR_CAPACITY;
        sp.v[b] = start_pos[b];
    }
    Shape s = shape_of(*d);
    cudaStream_t cs = (cudaStream_t)stream;
    if (s.bf16 && prefill_qm_supported(s))
        return launched(launch_prefill_qm(s, *q, *c, batch, seqlen, sp, out,
                                          device_error_ptr(), wait_limit(), cs));
    if (s.bf16 && prefill_tc_supported(s))
        return launched(launch_prefill_tc(s, *q, *c, batch, seqlen, sp, out,
                                          device_error_ptr(), wait_limit(), cs));
    return launched(launch_prefill_simt(s, *q, *c, batch, seqlen, sp, out, device_error_ptr(), cs));
}

size_t tpa_decode_workspace_bytes(const tpa_dims* d, const int32_t* lengths, int32_t batch) {
    if (check_dims(d, false) != TPA_OK || !lengths || batch < 1 || batch > TPA_MAX_BATCH)
        return 0;
    for (int b = 0; b < batch; ++b)
        if (lengths[b] < 1) return 0;
    Shape s = shape_of(*d);
    DecodePlan plan;
    make_decode_plan(s, lengths, batch, s.bf16 && decode_tc_supported(s), &plan);
    return decode_workspace_bytes(s, plan);
}

tpa_status tpa_decode(const tpa_dims* d, const void* q_a, const void* q_b,
                      const tpa_cache* c, const int32_t* lengths, int32_t batch, void* out,
                      void* workspace, size_t workspace_bytes, tpa_stream_t stream) {
    tpa_status st = tpa::validate_decode(d, q_a, q_b, c, lengths, batch, out);
    if (st != TPA_OK) return st;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return TPA_ERR_INVALID;
    return run_decode(shape_of(*d), q_a, q_b, *c, lengths, batch, out, workspace, workspace_bytes,
                      (cudaStream_t)stream);
}

tpa_status tpa_output_project(const tpa_dims* d, const void* attn, const void* w_o, int32_t T,
                              void* out, tpa_stream_t stream) {
    tpa_status st = check_dims(d, false);
    if (st != TPA_OK) return st;
    if (d->d_model < 1 || T < 1) return TPA_ERR_INVALID;
    if (!attn || !w_o || !out) return TPA_ERR_INVALID;
    if (!aligned16(attn) || !aligned16(w_o) || !aligned16(out)) return TPA_ERR_INVALID;
    if ((long long)d->n_heads * d->head_dim > (1 << 20) || T > (1 << 30)) return TPA_ERR_UNSUPPORTED;
    // the projection GEMM with one output segment (no RoPE pair in it): K = h*d_h
    Shape s = shape_of(*d);
    s.D = d->n_heads * d->head_dim;
    ProjLayout L;
    for (int i = 0; i < 6; ++i) L.off[i] = 0;
    L.off[6] = d->d_model;
    for (int i = 0; i < 6; ++i) { L.dst[i] = out; L.rows[i] = T; }
    SeqParams sp;
    sp.v[0] = 0;
    return run_project(s, attn, w_o, 1, T, sp, nullptr, L, (cudaStream_t)stream);
}

size_t tpa_decode_step_workspace_bytes(const tpa_dims* d, const int32_t* lengths, int32_t batch) {
    if (check_dims(d, false) != TPA_OK || !lengths || batch < 1 || batch > TPA_MAX_BATCH)
        return 0;
    int32_t next[TPA_MAX_BATCH];
    for (int b = 0; b < batch; ++b) {
        if (lengths[b] < 0) return 0;
        next[b] = lengths[b] + 1;
    }
    Shape s = shape_of(*d);
    DecodePlan plan;
    make_decode_plan(s, next, batch, s.bf16 && decode_tc_supported(s), &plan);
    return step_query_bytes(s, batch) + decode_workspace_bytes(s, plan);
}

tpa_status tpa_decode_step(const tpa_dims* d, const void* x, const void* w_cat,
                           const float* rope_cs, int32_t max_pos, const tpa_cache* c,
                           const int32_t* lengths, int32_t batch, void* out,
                           void* workspace, size_t workspace_bytes, tpa_stream_t stream) {
    tpa_status st = check_dims(d, false);
    if (st != TPA_OK) return st;
    if ((st = check_cache(c, batch)) != TPA_OK) return st;
    if (d->d_model < 1) return TPA_ERR_INVALID;
    if (!x || !w_cat || !rope_cs || !lengths || !out || !workspace) return TPA_ERR_INVALID;
    if (!aligned16(x) || !aligned16(w_cat) || !aligned16(rope_cs) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return TPA_ERR_INVALID;
    if ((d->n_heads * (d->rank_q + d->rank_k + d->rank_v)) & 1) return TPA_ERR_UNSUPPORTED;
    SeqParams sp;
    int32_t next[TPA_MAX_BATCH];
    for (int b = 0; b < batch; ++b) {
        if (lengths[b] < 0 || max_pos < 1) return TPA_ERR_INVALID;
        if (lengths[b] >= max_pos || lengths[b] + 1 > c->capacity) return TPA_ERR_CAPACITY;
        sp.v[b] = lengths[b];
        next[b] = lengths[b] + 1;
    }
    Shape s = shape_of(*d);
    const size_t qb = step_query_bytes(s, batch);
    if (workspace_bytes < qb) return TPA_ERR_WORKSPACE;
    // the new token's query factors go to the front of the workspace; its K/V factors
    // go straight into the cache rows lengths[b], and cache->lengths[b] is advanced
    const size_t es = s.bf16 ? 2 : 4;
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    const size_t aq_bytes = round_up((size_t)batch * s.H * s.Rq * es, 256);
    tpa_factors f;
    f.a_q = s.Rq > 0 ? wsb : nullptr;
    f.b_q = wsb + aq_bytes;
    f.a_k = c->a_k; f.a_v = c->a_v; f.b_k = c->b_k; f.b_v = c->b_v;
    ProjLayout L = proj_layout(s, f, batch, max_pos);
    L.kv_cap = c->capacity;
    L.lengths = c->lengths;
    L.n_lengths = c->batch;
    for (int i : {1, 2, 4, 5}) L.rows[i] = (long long)c->batch * c->capacity;
    cudaStream_t cs = (cudaStream_t)stream;
    // check the decode half before anything is launched
    {
        const bool tc = s.bf16 && decode_tc_supported(s);
        if (!tc && (long long)s.H * s.Dh > 8192) return TPA_ERR_UNSUPPORTED;
        DecodePlan plan;
        make_decode_plan(s, next, batch, tc, &plan);
        if (qb + decode_workspace_bytes(s, plan) > workspace_bytes) return TPA_ERR_WORKSPACE;
    }
    st = run_project(s, x, w_cat, batch, 1, sp, rope_cs, L, cs);
    if (st != TPA_OK) return st;
    return run_decode(s, f.a_q, f.b_q, *c, next, batch, out, wsb + qb, workspace_bytes - qb, cs);
}

int32_t tpa_kernel_family(const tpa_dims* d, int32_t call) {
    if (check_dims(d, false) != TPA_OK) return TPA_FAMILY_NONE;
    const Shape s = shape_of(*d);
    switch (call) {
        case TPA_CALL_PROJECT:
            return project_tc_supported(s, 1) ? TPA_FAMILY_TENSOR_CORE : TPA_FAMILY_CUDA_CORE;
        case TPA_CALL_PREFILL:
            if (d->head_dim > 256) return TPA_FAMILY_NONE;
            return s.bf16 && (prefill_qm_supported(s) || prefill_tc_supported(s)) ? TPA_FAMILY_TENSOR_CORE
                                                                                   : TPA_FAMILY_CUDA_CORE;
        case TPA_CALL_DECODE:
            if (s.bf16 && decode_tc_supported(s)) return TPA_FAMILY_TENSOR_CORE;
            return (long long)s.H * s.Dh > 8192 ? TPA_FAMILY_NONE : TPA_FAMILY_CUDA_CORE;
    }
    return TPA_FAMILY_NONE;
}

tpa_status tpa_get_device_error(tpa_stream_t stream, int32_t* code) {
    if (code) *code = 0;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return TPA_ERR_CUDA;
    int* p = device_error_ptr();
    if (!p) return TPA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return TPA_ERR_CUDA;
    if (v != 0) {
        int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return TPA_ERR_CUDA;
    }
    if (code) *code = v;
    return v ? TPA_ERR_DEVICE : TPA_OK;
}

}  // extern "C"
