// C ABI of the KDA library: argument validation (before any launch), workspace sizing and
// dispatch to the kernels.  See include/kda.h for the contract of every entry point.
#include <cstdint>
#include <cstring>
#include <vector>

#include "kda_common.cuh"

namespace {

constexpr size_t kStatusBytes = 256;  // status word + padding at the head of the workspace

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
};
Range range_of(const void *p, size_t bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + bytes};
}
bool overlaps(const Range &a, const Range &b) {
    return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi;
}

bool supported_dims(int dk, int dv) { return (dk == 128 && dv == 128) || (dk == 64 && dv == 64); }

bool uses_tensor_cores(int dk, int dv, kda_dtype dtype) {
    return dtype == KDA_BF16 && dk == 128 && dv == 128;
}

size_t elem_size(kda_dtype d) { return d == KDA_BF16 ? 2 : 4; }

// Shape checks common to the prefill entry points.  Returns KDA_OK or an error code.
int check_prefill_shape(int B, int T, int H, int dk, int dv, int num_seqs, bool varlen, int chunk) {
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || num_seqs <= 0) return KDA_ERR_BAD_SHAPE;
    if (varlen ? (B != 1) : (num_seqs != B)) return KDA_ERR_BAD_SHAPE;
    const int64_t tokens = (int64_t)B * T;
    if (tokens * H * (int64_t)(dk > dv ? dk : dv) > ((int64_t)1 << 40)) return KDA_ERR_BAD_SHAPE;
    if (tokens > INT32_MAX || (int64_t)num_seqs * H > INT32_MAX / 4) return KDA_ERR_BAD_SHAPE;
    if (chunk != kda::kChunk) return KDA_ERR_UNSUPPORTED;
    if (!supported_dims(dk, dv)) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

}  // namespace

// ------------------------------------------------------------------ per-kernel timing diagnostics
namespace kda {
namespace {
struct TraceState {
    bool on = false;
    int capacity = 0, used = 0;
    std::vector<cudaEvent_t> ev;  // 2 per kernel
    std::vector<int> ids;
};
TraceState g_trace;
}  // namespace

void trace_before(int kernel_id, cudaStream_t stream) {
    if (!g_trace.on || g_trace.used >= g_trace.capacity) return;
    g_trace.ids[g_trace.used] = kernel_id;
    cudaEventRecord(g_trace.ev[2 * g_trace.used], stream);
}
void trace_after(cudaStream_t stream) {
    if (!g_trace.on || g_trace.used >= g_trace.capacity) return;
    cudaEventRecord(g_trace.ev[2 * g_trace.used + 1], stream);
    ++g_trace.used;
}
}  // namespace kda

extern "C" {

int kda_trace_begin(int max_kernels) {
    using kda::g_trace;
    if (max_kernels <= 0) return KDA_ERR_BAD_SHAPE;
    if ((int)g_trace.ev.size() < 2 * max_kernels) {
        const size_t old = g_trace.ev.size();
        g_trace.ev.resize(2 * (size_t)max_kernels);
        for (size_t i = old; i < g_trace.ev.size(); ++i)
            if (cudaEventCreate(&g_trace.ev[i]) != cudaSuccess) {
                g_trace.ev.resize(i);
                return KDA_ERR_CUDA;
            }
    }
    g_trace.ids.assign(max_kernels, -1);
    g_trace.capacity = max_kernels;
    g_trace.used = 0;
    g_trace.on = true;
    return KDA_OK;
}

int kda_trace_end(int *kernel_ids, float *ms, int capacity) {
    using kda::g_trace;
    g_trace.on = false;
    if (cudaDeviceSynchronize() != cudaSuccess) return KDA_ERR_CUDA;
    const int n = g_trace.used;
    for (int i = 0; i < n && i < capacity; ++i) {
        float t = 0.f;
        if (cudaEventElapsedTime(&t, g_trace.ev[2 * i], g_trace.ev[2 * i + 1]) != cudaSuccess) return KDA_ERR_CUDA;
        if (kernel_ids) kernel_ids[i] = g_trace.ids[i];
        if (ms) ms[i] = t;
    }
    return n;
}


int kda_version(void) { return 100; }

const char *kda_status_string(int status) {
    switch (status) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_NULL_ARG: return "KDA_ERR_NULL_ARG: a required pointer is NULL";
        case KDA_ERR_BAD_SHAPE: return "KDA_ERR_BAD_SHAPE: a size is invalid or inconsistent";
        case KDA_ERR_BAD_DTYPE: return "KDA_ERR_BAD_DTYPE: unknown element type";
        case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED: a pointer is not 16-byte aligned";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: head dim or chunk size not implemented";
        case KDA_ERR_BAD_SEQLENS: return "KDA_ERR_BAD_SEQLENS: cu_seqlens is not 0..T non-decreasing";
        case KDA_ERR_WORKSPACE_TOO_SMALL: return "KDA_ERR_WORKSPACE_TOO_SMALL: workspace below the required size";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA runtime call failed";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device wait gave up";
        case KDA_ERR_ALIASING: return "KDA_ERR_ALIASING: an output overlaps an input";
        case KDA_ERR_BAD_SLOT: return "KDA_ERR_BAD_SLOT: a state-pool slot index is out of range";
        case KDA_ERR_BAD_VALUE: return "KDA_ERR_BAD_VALUE: a scalar argument is out of range";
        default: return "KDA: unknown status";
    }
}

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int chunk_size,
                                    kda_dtype dtype) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return 0;
    // Varlen-ness does not change validity here beyond B; size for the larger (varlen) table.
    const bool varlen = (B == 1 && num_seqs > 1);
    if (check_prefill_shape(B, T, H, dk, dv, num_seqs, varlen, chunk_size) != KDA_OK) return 0;
    // The tensor-core path's layout starts with the same 256-byte status block.
    if (uses_tensor_cores(dk, dv, dtype)) return kda::prefill_tc_workspace_bytes(B, T, H, num_seqs, true);
    return kStatusBytes;
}

// Checks the prologue arguments shared by the _ex entry points (A_log [H], dt_bias [H, dk]).
static int check_prologue(unsigned flags, const float *A_log, const float *dt_bias, int H, int dk, Range *ra, Range *rb) {
    if (flags & ~(unsigned)(KDA_PROLOGUE_L2NORM_QK | KDA_PROLOGUE_GATE)) return KDA_ERR_UNSUPPORTED;
    const bool gate = flags & KDA_PROLOGUE_GATE;
    if (gate && !A_log) return KDA_ERR_NULL_ARG;
    if (gate && (!aligned16(A_log) || (dt_bias && !aligned16(dt_bias)))) return KDA_ERR_MISALIGNED;
    *ra = range_of(A_log, gate ? (size_t)H * 4 : 0);
    *rb = range_of(dt_bias, gate && dt_bias ? (size_t)H * dk * 4 : 0);
    return KDA_OK;
}

int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                  const float *h0, const int32_t *cu_seqlens, int num_seqs, int B, int T, int H, int dk,
                  int dv, int chunk_size, kda_dtype dtype, void *o, float *h_T, void *workspace,
                  size_t workspace_bytes, void *stream) {
    return kda_chunk_fwd_ex(q, k, v, log_alpha, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv, chunk_size, dtype,
                            o, h_T, workspace, workspace_bytes, 0u, nullptr, nullptr, stream);
}

int kda_chunk_fwd_ex(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                     const float *h0, const int32_t *cu_seqlens, int num_seqs, int B, int T, int H, int dk,
                     int dv, int chunk_size, kda_dtype dtype, void *o, float *h_T, void *workspace,
                     size_t workspace_bytes, unsigned flags, const float *A_log, const float *dt_bias,
                     void *stream_) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_BAD_DTYPE;
    if (!workspace) return KDA_ERR_NULL_ARG;
    const bool varlen = cu_seqlens != nullptr;
    int rc = check_prefill_shape(B, T, H, dk, dv, num_seqs, varlen, chunk_size);
    if (rc != KDA_OK) return rc;
    // with no tokens the token tensors are empty (never read) and may be NULL
    if ((int64_t)B * T > 0 && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_NULL_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, beta, h0, cu_seqlens, o, h_T};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_MISALIGNED;

    const size_t es = elem_size(dtype);
    const size_t tok = (size_t)B * T * H;
    const size_t sbytes = (size_t)num_seqs * H * dk * dv * sizeof(float);
    const Range ro = range_of(o, tok * dv * es);
    const Range inputs[] = {range_of(q, tok * dk * es), range_of(k, tok * dk * es), range_of(v, tok * dv * es),
                            range_of(log_alpha, tok * dk * 4), range_of(beta, tok * 4),
                            range_of(h0, h0 ? sbytes : 0),
                            range_of(cu_seqlens, cu_seqlens ? (size_t)(num_seqs + 1) * 4 : 0)};
    for (const Range &r : inputs)
        if (overlaps(ro, r)) return KDA_ERR_ALIASING;
    if (h_T) {
        const Range rh = range_of(h_T, sbytes);
        if (overlaps(rh, ro)) return KDA_ERR_ALIASING;
        for (int i = 0; i < 5; ++i)
            if (overlaps(rh, inputs[i])) return KDA_ERR_ALIASING;
        if (overlaps(rh, inputs[6])) return KDA_ERR_ALIASING;
        if (h0 && h_T != h0 && overlaps(rh, inputs[5])) return KDA_ERR_ALIASING;
    }
    Range ra, rb;
    if ((rc = check_prologue(flags, A_log, dt_bias, H, dk, &ra, &rb)) != KDA_OK) return rc;
    if (overlaps(ro, ra) || overlaps(ro, rb)) return KDA_ERR_ALIASING;
    if (h_T && (overlaps(range_of(h_T, sbytes), ra) || overlaps(range_of(h_T, sbytes), rb))) return KDA_ERR_ALIASING;
    const kda::Prologue pro{flags, A_log, dt_bias};
    const size_t need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs, chunk_size, dtype);
    if (need == 0) return KDA_ERR_BAD_SHAPE;
    if (workspace_bytes < need) return KDA_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    int *status = static_cast<int *>(workspace);
    cudaError_t e;
    if (uses_tensor_cores(dk, dv, dtype)) {
        e = kda::launch_prefill_tc(q, k, v, log_alpha, beta, h0, cu_seqlens, num_seqs, B, T, H, o, h_T,
                                   workspace, workspace_bytes, pro, stream);
    } else {
        e = cudaMemsetAsync(workspace, 0, kStatusBytes, stream);
        if (e == cudaSuccess)
            e = kda::launch_prefill_simt(q, k, v, log_alpha, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv,
                                     dtype, o, h_T, status, pro, stream);
    }
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                    float *S, int N, int H, int dk, int dv, kda_dtype dtype, void *o, void *stream_) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_BAD_DTYPE;
    if (!q || !k || !v || !log_alpha || !beta || !S || !o) return KDA_ERR_NULL_ARG;
    if (N <= 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_BAD_SHAPE;
    if ((int64_t)N * H > (int64_t)INT32_MAX) return KDA_ERR_BAD_SHAPE;
    if (!supported_dims(dk, dv)) return KDA_ERR_UNSUPPORTED;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_MISALIGNED;
    const size_t es = elem_size(dtype), units = (size_t)N * H;
    const Range ro = range_of(o, units * dv * es), rs = range_of(S, units * dk * dv * 4);
    const Range inputs[] = {range_of(q, units * dk * es), range_of(k, units * dk * es),
                            range_of(v, units * dv * es), range_of(log_alpha, units * dk * 4),
                            range_of(beta, units * 4)};
    if (overlaps(ro, rs)) return KDA_ERR_ALIASING;
    for (const Range &r : inputs)
        if (overlaps(ro, r) || overlaps(rs, r)) return KDA_ERR_ALIASING;
    cudaError_t e = kda::launch_decode(q, k, v, log_alpha, beta, S, N, H, dk, dv, dtype, o,
                                       static_cast<cudaStream_t>(stream_));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_decode_multi(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                     float *S_pool, int num_slots, const int32_t *slot_in, const int32_t *slot_out, int N, int Tq,
                     int H, int dk, int dv, kda_dtype dtype, void *o, int *status, void *stream) {
    return kda_decode_multi_ex(q, k, v, log_alpha, beta, S_pool, num_slots, slot_in, slot_out, N, Tq, H, dk, dv,
                               dtype, o, status, 0u, nullptr, nullptr, stream);
}

int kda_decode_multi_ex(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                        float *S_pool, int num_slots, const int32_t *slot_in, const int32_t *slot_out, int N,
                        int Tq, int H, int dk, int dv, kda_dtype dtype, void *o, int *status, unsigned flags,
                        const float *A_log, const float *dt_bias, void *stream_) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_BAD_DTYPE;
    if (!q || !k || !v || !log_alpha || !beta || !S_pool || !o) return KDA_ERR_NULL_ARG;
    if (N <= 0 || Tq <= 0 || H <= 0 || dk <= 0 || dv <= 0 || num_slots <= 0) return KDA_ERR_BAD_SHAPE;
    const int64_t tokens = (int64_t)N * Tq * H, states = (int64_t)num_slots * H;
    if ((int64_t)N * H > (int64_t)INT32_MAX || tokens * (dk > dv ? dk : dv) > ((int64_t)1 << 40) ||
        states * dk * dv > ((int64_t)1 << 40))
        return KDA_ERR_BAD_SHAPE;
    if ((!slot_in || !slot_out) && N > num_slots) return KDA_ERR_BAD_SHAPE;  // slot n must exist
    if (!supported_dims(dk, dv)) return KDA_ERR_UNSUPPORTED;
    const void *ptrs[] = {q, k, v, log_alpha, beta, S_pool, o};
    for (const void *p : ptrs)
        if (!aligned16(p)) return KDA_ERR_MISALIGNED;
    const void *words[] = {slot_in, slot_out, status};
    for (const void *p : words)
        if (reinterpret_cast<uintptr_t>(p) % 4 != 0) return KDA_ERR_MISALIGNED;
    const size_t es = elem_size(dtype);
    const Range ro = range_of(o, (size_t)tokens * dv * es), rs = range_of(S_pool, (size_t)states * dk * dv * 4),
                rst = range_of(status, status ? 4 : 0);
    const Range inputs[] = {range_of(q, (size_t)tokens * dk * es), range_of(k, (size_t)tokens * dk * es),
                            range_of(v, (size_t)tokens * dv * es), range_of(log_alpha, (size_t)tokens * dk * 4),
                            range_of(beta, (size_t)tokens * 4), range_of(slot_in, slot_in ? (size_t)N * 4 : 0),
                            range_of(slot_out, slot_out ? (size_t)N * 4 : 0)};
    if (overlaps(ro, rs) || overlaps(ro, rst) || overlaps(rs, rst)) return KDA_ERR_ALIASING;
    for (const Range &r : inputs)
        if (overlaps(ro, r) || overlaps(rs, r) || overlaps(rst, r)) return KDA_ERR_ALIASING;
    Range ra, rb;
    const int prc = check_prologue(flags, A_log, dt_bias, H, dk, &ra, &rb);
    if (prc != KDA_OK) return prc;
    if (overlaps(ro, ra) || overlaps(ro, rb) || overlaps(rs, ra) || overlaps(rs, rb) || overlaps(rst, ra) ||
        overlaps(rst, rb))
        return KDA_ERR_ALIASING;
    const kda::Prologue pro{flags, A_log, dt_bias};
    cudaError_t e = kda::launch_decode_multi(q, k, v, log_alpha, beta, S_pool, num_slots, slot_in, slot_out, N, Tq,
                                             H, dk, dtype, o, status, pro, static_cast<cudaStream_t>(stream_));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int chunk_size,
                                    kda_dtype dtype) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return 0;
    const bool varlen = (B == 1 && num_seqs > 1);
    if (check_prefill_shape(B, T, H, dk, dv, num_seqs, varlen, chunk_size) != KDA_OK) return 0;
    if (dk != dv) return 0;
    return kda::chunk_bwd_workspace_bytes(B, T, H, dk, num_seqs, dtype);
}

int kda_chunk_bwd(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                  const float *h0, const int32_t *cu_seqlens, int num_seqs, int B, int T, int H, int dk, int dv,
                  int chunk_size, kda_dtype dtype, const void *do_, const float *dh_T, void *dq, void *dk_out,
                  void *dv_out, float *dlog_alpha, float *dbeta, float *dh0, void *workspace, size_t workspace_bytes,
                  void *stream_) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_BAD_DTYPE;
    if (!workspace) return KDA_ERR_NULL_ARG;
    const int rc = check_prefill_shape(B, T, H, dk, dv, num_seqs, cu_seqlens != nullptr, chunk_size);
    if (rc != KDA_OK) return rc;
    if (dk != dv) return KDA_ERR_UNSUPPORTED;
    const int64_t tokens = (int64_t)B * T;
    if (tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !do_ || !dq || !dk_out || !dv_out || !dlog_alpha ||
                       !dbeta))
        return KDA_ERR_NULL_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, beta, h0, do_, dh_T, dq, dk_out, dv_out, dlog_alpha, dbeta, dh0};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_MISALIGNED;
    const size_t need = kda::chunk_bwd_workspace_bytes(B, T, H, dk, num_seqs, dtype);
    if (workspace_bytes < need) return KDA_ERR_WORKSPACE_TOO_SMALL;
    const size_t es = elem_size(dtype), tk = (size_t)tokens * H, sb = (size_t)num_seqs * H * dk * dv * 4;
    const Range in[] = {range_of(q, tk * dk * es), range_of(k, tk * dk * es), range_of(v, tk * dv * es),
                        range_of(log_alpha, tk * dk * 4), range_of(beta, tk * 4), range_of(h0, h0 ? sb : 0),
                        range_of(do_, tk * dv * es), range_of(dh_T, dh_T ? sb : 0),
                        range_of(cu_seqlens, cu_seqlens ? 4 * (size_t)(num_seqs + 1) : 0)};
    const Range out[] = {range_of(dq, tk * dk * es), range_of(dk_out, tk * dk * es), range_of(dv_out, tk * dv * es),
                         range_of(dlog_alpha, tk * dk * 4), range_of(dbeta, tk * 4), range_of(dh0, dh0 ? sb : 0),
                         range_of(workspace, need)};
    for (size_t a = 0; a < sizeof(out) / sizeof(out[0]); ++a) {
        for (const Range &r : in)
            if (overlaps(out[a], r)) return KDA_ERR_ALIASING;
        for (size_t b = a + 1; b < sizeof(out) / sizeof(out[0]); ++b)
            if (overlaps(out[a], out[b])) return KDA_ERR_ALIASING;
    }
    if (tokens == 0) {  // nothing to differentiate but the initial states: dh0 = dh_T
        cudaStream_t st = static_cast<cudaStream_t>(stream_);
        cudaError_t e = cudaSuccess;
        if (dh0) e = dh_T ? cudaMemcpyAsync(dh0, dh_T, sb, cudaMemcpyDeviceToDevice, st) : cudaMemsetAsync(dh0, 0, sb, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, 256, st);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    cudaError_t e = kda::launch_chunk_bwd(q, k, v, log_alpha, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dtype, do_,
                                          dh_T, dq, dk_out, dv_out, dlog_alpha, dbeta, dh0, workspace,
                                          static_cast<cudaStream_t>(stream_));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_state_compose(const float *Mb, const float *h0, int R, int H, int dk, int dv, float *S_in, float *S_out,
                      void *stream_) {
    if (!Mb || !S_out) return KDA_ERR_NULL_ARG;
    if (R <= 0 || H <= 0 || dk <= 0 || dv <= 0 || (int64_t)R * H * dk * (dk + dv) > ((int64_t)1 << 40))
        return KDA_ERR_BAD_SHAPE;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return KDA_ERR_UNSUPPORTED;
    const void *ptrs[] = {Mb, h0, S_in, S_out};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    const size_t sb = (size_t)H * dk * dv * 4;
    const Range rm = range_of(Mb, (size_t)R * H * dk * (dk + dv) * 4), rh = range_of(h0, h0 ? sb : 0),
                ri = range_of(S_in, S_in ? (size_t)R * sb : 0), ro = range_of(S_out, sb);
    if (overlaps(ro, rm) || overlaps(ro, rh) || overlaps(ro, ri) || overlaps(ri, rm) || overlaps(ri, rh))
        return KDA_ERR_ALIASING;
    cudaError_t e = kda::launch_state_compose(Mb, h0, R, H, dk, dv, S_in, S_out, static_cast<cudaStream_t>(stream_));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_segment_map(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta, int T,
                    int H, int dk, int dv, int chunk_size, kda_dtype dtype, void *o0, float *Mb, void *workspace,
                    size_t workspace_bytes, void *stream_) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_BAD_DTYPE;
    if (!workspace || !Mb) return KDA_ERR_NULL_ARG;
    int rc = check_prefill_shape(1, T, H, dk, dv, 1, false, chunk_size);
    if (rc != KDA_OK) return rc;
    if (!uses_tensor_cores(dk, dv, dtype)) return KDA_ERR_UNSUPPORTED;
    if (T > 0 && (!q || !k || !v || !log_alpha || !beta)) return KDA_ERR_NULL_ARG;
    const void *ptrs[] = {q, k, v, log_alpha, beta, o0, Mb};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_MISALIGNED;
    const size_t es = elem_size(dtype), tok = (size_t)T * H;
    const size_t need = kda_chunk_fwd_workspace_size(1, T, H, dk, dv, 1, chunk_size, dtype);
    if (need == 0) return KDA_ERR_BAD_SHAPE;
    if (workspace_bytes < need) return KDA_ERR_WORKSPACE_TOO_SMALL;
    const Range rm = range_of(Mb, (size_t)H * dk * (dk + dv) * 4), ro = range_of(o0, o0 ? tok * dv * es : 0),
                rw = range_of(workspace, need);
    const Range inputs[] = {range_of(q, tok * dk * es), range_of(k, tok * dk * es), range_of(v, tok * dv * es),
                            range_of(log_alpha, tok * dk * 4), range_of(beta, tok * 4)};
    if (overlaps(rm, ro) || overlaps(rm, rw) || overlaps(ro, rw)) return KDA_ERR_ALIASING;
    for (const Range &r : inputs)
        if (overlaps(rm, r) || overlaps(ro, r)) return KDA_ERR_ALIASING;
    const kda::Prologue pro{0u, nullptr, nullptr};
    cudaError_t e = kda::launch_prefill_tc(q, k, v, log_alpha, beta, nullptr, nullptr, 1, 1, T, H, o0, nullptr,
                                           workspace, workspace_bytes, pro, static_cast<cudaStream_t>(stream_), Mb);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_output_gate_norm(const void *o, const void *g, const float *weight, float eps, int n_tok, int H, int dv,
                         kda_dtype dtype, void *out, void *stream_) {
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_BAD_DTYPE;
    if (n_tok < 0 || H <= 0 || dv <= 0) return KDA_ERR_BAD_SHAPE;
    const int64_t rows = (int64_t)n_tok * H;
    if (rows * dv > ((int64_t)1 << 40)) return KDA_ERR_BAD_SHAPE;
    if (dv != 64 && dv != 128) return KDA_ERR_UNSUPPORTED;
    if (!(eps >= 0.f) || eps > 3.0e38f) return KDA_ERR_BAD_VALUE;
    if (rows == 0) return KDA_OK;
    if (!o || !g || !out) return KDA_ERR_NULL_ARG;
    const void *ptrs[] = {o, g, out, weight};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
    const size_t bytes = (size_t)rows * dv * elem_size(dtype);
    const Range ro = range_of(o, bytes), rg = range_of(g, bytes), rw = range_of(weight, weight ? (size_t)dv * 4 : 0),
                rout = range_of(out, bytes);
    if (out != o && overlaps(rout, ro)) return KDA_ERR_ALIASING;
    if (overlaps(rout, rg) || overlaps(rout, rw)) return KDA_ERR_ALIASING;
    cudaError_t e = kda::launch_output_gate_norm(o, g, weight, eps, rows, dv, dtype, out,
                                                 static_cast<cudaStream_t>(stream_));
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int kda_get_status(void *workspace, void *stream_) {
    if (!workspace) return KDA_ERR_NULL_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    int host = 0;
    if (cudaMemcpyAsync(&host, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    if (host != 0) {
        const int zero = 0;
        if (cudaMemcpyAsync(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return KDA_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    }
    return host;
}

}  // extern "C"
