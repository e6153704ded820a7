// kda_api.cu -- the C ABI of libkda_b200.so (declared in include/kda.h).
//
// Host side only: argument validation, kernel selection and launch on the
// caller's stream.  The whole library is this one translation unit; the
// kernels live in the headers included below.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/kda.h"
#include "kda_backward.cuh"
#include "kda_chunk_tc.cuh"
#include "kda_common.cuh"
#include "kda_decode.cuh"
#include "kda_recurrent.cuh"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool head_ok(int d) { return d == 64 || d == 128; }

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// Checks shared by kda_chunk_fwd and kda_recurrent_fwd.  Returns KDA_OK when
// the call is well-formed.
kda_status check_prefill(const void *q, const void *k, const void *v, const void *la, const void *beta,
                         const float *init_state, const int32_t *cu, int32_t num_seqs, int32_t B, int32_t T,
                         int32_t H, int32_t dk, int32_t dv, kda_dtype dtype, kda_dtype out_dtype,
                         const void *out, const float *final_state, int gate) {
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return KDA_ERR_INVALID_ARG;
    // token tensors may be empty (NULL) only when there are no tokens; a per-head gate may be NULL
    // (no decay)
    if (T > 0 && (!q || !k || !v || (gate != kda::kGateHead && !la) || !beta || !out))
        return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (out_dtype != KDA_F32 && out_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (cu) {
        if (B != 1 || num_seqs < 1) return KDA_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(cu) & 3u) != 0) return KDA_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {q, k, v, la, beta, out, init_state, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    // an in-place state update must alias exactly
    if (init_state && final_state && init_state != final_state) {
        const int64_t N = cu ? num_seqs : B;
        const size_t bytes = (size_t)N * H * dk * dv * sizeof(float);
        const char *a = reinterpret_cast<const char *>(init_state), *b = reinterpret_cast<const char *>(final_state);
        if (a < b + bytes && b < a + bytes) return KDA_ERR_INVALID_ARG;
    }
    // 64-bit element counts must stay addressable by the kernels' index math
    const int64_t tokens = (int64_t)B * T * H;
    if (tokens * (dk > dv ? dk : dv) > (int64_t(1) << 46)) return KDA_ERR_UNSUPPORTED;
    if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
    const int64_t ctas = (int64_t)(cu ? num_seqs : B) * H * (dv / 32);
    if (ctas > 0x7fffffff) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

template <typename TIO, typename TOUT, int GK>
cudaError_t dispatch_recurrent_g(const void *q, const void *k, const void *v, const void *la, const void *beta,
                                 const float *s0, const int32_t *cu, int ns, int B, int T, int H, int dk, int dv,
                                 void *out, float *fs, cudaStream_t st) {
    if (dk == 64)
        return kda::launch_recurrent<64, TIO, TOUT, GK>(q, k, v, la, beta, s0, cu, ns, B, T, H, dv, out, fs, st);
    return kda::launch_recurrent<128, TIO, TOUT, GK>(q, k, v, la, beta, s0, cu, ns, B, T, H, dv, out, fs, st);
}

template <typename TIO, typename TOUT>
cudaError_t dispatch_recurrent_t(int gate, const void *q, const void *k, const void *v, const void *la,
                                 const void *beta, const float *s0, const int32_t *cu, int ns, int B, int T, int H,
                                 int dk, int dv, void *out, float *fs, cudaStream_t st) {
    if (gate == kda::kGateHead)
        return dispatch_recurrent_g<TIO, TOUT, kda::kGateHead>(q, k, v, la, beta, s0, cu, ns, B, T, H, dk, dv, out,
                                                               fs, st);
    return dispatch_recurrent_g<TIO, TOUT, kda::kGateChannel>(q, k, v, la, beta, s0, cu, ns, B, T, H, dk, dv, out,
                                                              fs, st);
}

cudaError_t dispatch_recurrent(int gate, kda_dtype dt, kda_dtype odt, const void *q, const void *k,
                               const void *v, const void *la, const void *beta, const float *s0, const int32_t *cu,
                               int ns, int B, int T, int H, int dk, int dv, void *out, float *fs, cudaStream_t st) {
    if (dt == KDA_F32 && odt == KDA_F32)
        return dispatch_recurrent_t<float, float>(gate, q, k, v, la, beta, s0, cu, ns, B, T, H, dk, dv, out, fs, st);
    if (dt == KDA_F32)
        return dispatch_recurrent_t<float, __nv_bfloat16>(gate, q, k, v, la, beta, s0, cu, ns, B, T, H, dk, dv, out,
                                                          fs, st);
    if (odt == KDA_F32)
        return dispatch_recurrent_t<__nv_bfloat16, float>(gate, q, k, v, la, beta, s0, cu, ns, B, T, H, dk, dv, out,
                                                          fs, st);
    return dispatch_recurrent_t<__nv_bfloat16, __nv_bfloat16>(gate, q, k, v, la, beta, s0, cu, ns, B, T, H, dk, dv,
                                                              out, fs, st);
}

// Handoff buffer of kda_chunk_fwd_static_ws: a fixed array in device memory,
// one copy per GPU that loads the library.  In host code `g_static_ws` only
// names the symbol; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_static_ws[KDA_STATIC_WS_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mutex;
void *g_static_ws_addr[kMaxDevices] = {};

// Device address of the current device's copy of g_static_ws.  It is looked up with that device
// current and cached per device.  Outside stream capture it is looked up again on every call (a
// cheap runtime query), so that a cached address never outlives a device reset; during capture
// the cached address is used, because the lookup may load the module, which capture forbids.
kda_status static_ws_address(void **addr, cudaStream_t stream) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_ws_mutex);
    if (cs == cudaStreamCaptureStatusNone || !g_static_ws_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) return KDA_ERR_CUDA;
        g_static_ws_addr[dev] = p;
    }
    *addr = g_static_ws_addr[dev];
    return KDA_OK;
}

}  // namespace

extern "C" {

const char *kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
    }
    return "KDA_ERR_UNKNOWN";
}

const char *kda_version(void) { return "kda_b200 0.2.0 sm_100a"; }

kda_status kda_testing_set_chunk_fault(int32_t skip_item, uint32_t flag_wait_us) {
    if (skip_item < -1) return KDA_ERR_INVALID_ARG;
    kda::ChunkFault &f = kda::chunk_fault();
    f.skip_item = skip_item;
    f.flag_wait_ns = flag_wait_us ? (uint64_t)flag_wait_us * 1000u : kda::tc::kFlagWaitNs;
    return KDA_OK;
}

kda_status kda_get_last_device_error(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return KDA_ERR_CUDA;
    int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, kda::g_device_error, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemcpyToSymbol(kda::g_device_error, &zero, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
    return word == 0 ? KDA_OK : static_cast<kda_status>(word);
}

}  // extern "C"

namespace {

kda_status recurrent_impl(int gate, const void *q, const void *k, const void *v, const void *la, const void *beta,
                          const float *init_state, const int32_t *cu_seqlens, int32_t num_seqs, int32_t B,
                          int32_t T, int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype, kda_dtype out_dtype,
                          void *out, float *final_state, void *stream) {
    kda_status s = check_prefill(q, k, v, la, beta, init_state, cu_seqlens, num_seqs, B, T, H, d_k, d_v, dtype,
                                 out_dtype, out, final_state, gate);
    if (s != KDA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return from_cuda(dispatch_recurrent(gate, dtype, out_dtype, q, k, v, la, beta, init_state, cu_seqlens, num_seqs,
                                        B, T, H, d_k, d_v, out, final_state, st));
}

// Shared by kda_chunk_fwd / gdn_chunk_fwd (workspace != NULL) and kda_chunk_fwd_static_ws
// (workspace == NULL: the built-in array).
kda_status chunk_impl(int gate, bool static_ws, const void *q, const void *k, const void *v, const void *la,
                      const void *beta, const float *init_state, const int32_t *cu_seqlens, int32_t num_seqs,
                      int32_t B, int32_t T, int32_t H, int32_t d_k, int32_t d_v, int32_t chunk, kda_dtype dtype,
                      kda_dtype out_dtype, void *out, float *final_state, void *workspace, size_t workspace_bytes,
                      void *stream) {
    kda_status s = check_prefill(q, k, v, la, beta, init_state, cu_seqlens, num_seqs, B, T, H, d_k, d_v, dtype,
                                 out_dtype, out, final_state, gate);
    if (s != KDA_OK) return s;
    if (chunk < 1) return KDA_ERR_INVALID_ARG;
    // chunks of up to 64 tokens (the tensor-core kernel's tile height); 128 would need a larger image
    // than the chain's shared memory holds three of
    if (chunk > kda::kChunk) return KDA_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (static_ws || gate == kda::kRawInputs) {
        // the raw-projection form runs on the tensor-core path only
        if (dtype != KDA_BF16) return KDA_ERR_UNSUPPORTED;
    } else if (dtype == KDA_F32) {
        // fp32 I/O asks for fp32 accuracy, which bf16 tensor-core operands
        // cannot give: evaluate on CUDA cores with the fp32 state.
        return from_cuda(dispatch_recurrent(gate, dtype, out_dtype, q, k, v, la, beta, init_state, cu_seqlens,
                                            num_seqs, B, T, H, d_k, d_v, out, final_state, st));
    }
    if ((int64_t)B * T >= (int64_t(1) << 31)) return KDA_ERR_UNSUPPORTED;   // 32-bit token coordinates
    const int64_t pairs = (int64_t)(cu_seqlens ? num_seqs : B) * H;
    if (static_ws) {
        // the schedule tables and rings of at least kMinRing images for each chain always fit
        const int64_t chains = pairs < kda::kMaxChains ? pairs : kda::kMaxChains;
        if (kda::flags_region_bytes() + (size_t)chains * kda::kMinRing * kda::img_stride(d_v) > KDA_STATIC_WS_BYTES)
            return KDA_ERR_UNSUPPORTED;
        s = static_ws_address(&workspace, st);
        if (s != KDA_OK) return s;
        workspace_bytes = KDA_STATIC_WS_BYTES;
    } else {
        const size_t need = kda::chunk_tc_workspace_bytes(pairs, d_v);
        if (!workspace || workspace_bytes < need || !aligned16(workspace)) return KDA_ERR_INVALID_ARG;
    }
    if (out_dtype == KDA_F32)
        return from_cuda(kda::launch_chunk_tc<float>(q, k, v, la, beta, init_state, cu_seqlens, num_seqs, B, T, H,
                                                     d_k, d_v, chunk, out, final_state, workspace, workspace_bytes,
                                                     st, gate));
    return from_cuda(kda::launch_chunk_tc<__nv_bfloat16>(q, k, v, la, beta, init_state, cu_seqlens, num_seqs, B, T,
                                                         H, d_k, d_v, chunk, out, final_state, workspace,
                                                         workspace_bytes, st, gate));
}

template <int GK>
kda_status decode_impl(const void *q, const void *k, const void *v, const void *la, const void *beta, float *state,
                       void *out, int32_t B, int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype,
                       kda_dtype out_dtype, void *stream) {
    if (!q || !k || !v || (GK != kda::kGateHead && !la) || !beta || !state || !out) return KDA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || d_k < 1 || d_v < 1) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (out_dtype != KDA_F32 && out_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    const void *ptrs[] = {q, k, v, la, beta, state, out};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (!head_ok(d_k) || !head_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)B * H > 0x7fffffff) return KDA_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
#define KDA_DECODE_CASE(DK, DV)                                                                                 \
    if (d_k == DK && d_v == DV) {                                                                               \
        if (dtype == KDA_F32)                                                                                   \
            e = out_dtype == KDA_F32                                                                            \
                    ? kda::launch_decode<DK, DV, float, float, GK>(q, k, v, la, beta, state, out, B, H, st)     \
                    : kda::launch_decode<DK, DV, float, __nv_bfloat16, GK>(q, k, v, la, beta, state, out, B, H, \
                                                                           st);                                 \
        else                                                                                                    \
            e = out_dtype == KDA_F32                                                                            \
                    ? kda::launch_decode<DK, DV, __nv_bfloat16, float, GK>(q, k, v, la, beta, state, out, B, H, \
                                                                           st)                                  \
                    : kda::launch_decode<DK, DV, __nv_bfloat16, __nv_bfloat16, GK>(q, k, v, la, beta, state,    \
                                                                                   out, B, H, st);              \
        return from_cuda(e);                                                                                    \
    }
    KDA_DECODE_CASE(128, 128)
    KDA_DECODE_CASE(128, 64)
    KDA_DECODE_CASE(64, 128)
    KDA_DECODE_CASE(64, 64)
#undef KDA_DECODE_CASE
    return KDA_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

kda_status kda_recurrent_fwd(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                             const float *init_state, const int32_t *cu_seqlens, int32_t num_seqs, int32_t B,
                             int32_t T, int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype,
                             kda_dtype out_dtype, void *out, float *final_state, void *stream) {
    return recurrent_impl(kda::kGateChannel, q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, B, T, H, d_k,
                          d_v, dtype, out_dtype, out, final_state, stream);
}

kda_status kda_chunk_fwd_workspace_size(int32_t N, int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype,
                                        size_t *bytes) {
    if (!bytes || N < 1 || H < 1) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    *bytes = 0;
    if (!head_ok(d_k) || !head_ok(d_v)) return KDA_ERR_UNSUPPORTED;
    if (dtype == KDA_BF16) *bytes = kda::chunk_tc_workspace_bytes((int64_t)N * H, d_v);
    return KDA_OK;
}

kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                         const float *init_state, const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                         int32_t H, int32_t d_k, int32_t d_v, int32_t chunk, kda_dtype dtype,
                         kda_dtype out_dtype, void *out, float *final_state, void *workspace, size_t workspace_bytes,
                         void *stream) {
    return chunk_impl(kda::kGateChannel, false, q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, B, T, H,
                      d_k, d_v, chunk, dtype, out_dtype, out, final_state, workspace, workspace_bytes, stream);
}

kda_status kda_chunk_fwd_static_ws(const void *q, const void *k, const void *v, const void *log_alpha,
                                   const void *beta, const float *init_state, const int32_t *cu_seqlens,
                                   int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                   int32_t chunk, kda_dtype dtype, kda_dtype out_dtype, void *out,
                                   float *final_state, void *stream) {
    return chunk_impl(kda::kGateChannel, true, q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, B, T, H,
                      d_k, d_v, chunk, dtype, out_dtype, out, final_state, nullptr, 0, stream);
}

kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                           float *state, void *out, int32_t B, int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype,
                           kda_dtype out_dtype, void *stream) {
    return decode_impl<kda::kGateChannel>(q, k, v, log_alpha, beta, state, out, B, H, d_k, d_v, dtype, out_dtype,
                                          stream);
}

kda_status gdn_chunk_fwd(const void *q, const void *k, const void *v, const void *log_g, const void *beta,
                         const float *init_state, const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                         int32_t H, int32_t d_k, int32_t d_v, int32_t chunk, kda_dtype dtype,
                         kda_dtype out_dtype, void *out, float *final_state, void *workspace, size_t workspace_bytes,
                         void *stream) {
    return chunk_impl(kda::kGateHead, false, q, k, v, log_g, beta, init_state, cu_seqlens, num_seqs, B, T, H, d_k,
                      d_v, chunk, dtype, out_dtype, out, final_state, workspace, workspace_bytes, stream);
}

kda_status gdn_recurrent_fwd(const void *q, const void *k, const void *v, const void *log_g, const void *beta,
                             const float *init_state, const int32_t *cu_seqlens, int32_t num_seqs, int32_t B,
                             int32_t T, int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype,
                             kda_dtype out_dtype, void *out, float *final_state, void *stream) {
    return recurrent_impl(kda::kGateHead, q, k, v, log_g, beta, init_state, cu_seqlens, num_seqs, B, T, H, d_k, d_v,
                          dtype, out_dtype, out, final_state, stream);
}

kda_status kda_chunk_fwd_fused(const void *q_raw, const void *k_raw, const void *v, const void *g_raw,
                               const void *b_raw, const float *init_state, const int32_t *cu_seqlens,
                               int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                               int32_t chunk, kda_dtype dtype, kda_dtype out_dtype, void *out, float *final_state,
                               void *workspace, size_t workspace_bytes, void *stream) {
    return chunk_impl(kda::kRawInputs, false, q_raw, k_raw, v, g_raw, b_raw, init_state, cu_seqlens, num_seqs, B, T,
                      H, d_k, d_v, chunk, dtype, out_dtype, out, final_state, workspace, workspace_bytes, stream);
}

kda_status kda_decode_step_fused(const void *q_raw, const void *k_raw, const void *v, const void *g_raw,
                                 const void *b_raw, float *state, void *out, int32_t B, int32_t H, int32_t d_k,
                                 int32_t d_v, kda_dtype dtype, kda_dtype out_dtype, void *stream) {
    return decode_impl<kda::kRawInputs>(q_raw, k_raw, v, g_raw, b_raw, state, out, B, H, d_k, d_v, dtype, out_dtype,
                                        stream);
}

kda_status gdn_decode_step(const void *q, const void *k, const void *v, const void *log_g, const void *beta,
                           float *state, void *out, int32_t B, int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype,
                           kda_dtype out_dtype, void *stream) {
    return decode_impl<kda::kGateHead>(q, k, v, log_g, beta, state, out, B, H, d_k, d_v, dtype, out_dtype, stream);
}

}  // extern "C"

extern "C" {

kda_status kda_chunk_bwd_workspace_size(int32_t N, int32_t H, int64_t total_tokens, int32_t d_k, int32_t d_v,
                                        int32_t chunk, size_t *bytes) {
    if (!bytes || N < 1 || H < 1 || total_tokens < 0 || chunk < 0) return KDA_ERR_INVALID_ARG;
    *bytes = 0;
    if (!head_ok(d_k) || !head_ok(d_v) || chunk > 256) return KDA_ERR_UNSUPPORTED;
    *bytes = kda::bwd_workspace_bytes(N, H, total_tokens, d_k, d_v, chunk);
    return KDA_OK;
}

kda_status kda_chunk_bwd(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                         const float *init_state, const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                         int32_t H, int32_t d_k, int32_t d_v, int32_t chunk, kda_dtype dtype, const void *d_out,
                         kda_dtype d_out_dtype, const float *d_final_state, float *dq, float *dk, float *dv,
                         float *dlog_alpha, float *dbeta, float *d_init_state, void *workspace,
                         size_t workspace_bytes, void *stream) {
    // the forward arguments are checked as for the prefill (d_out plays the part of `out`)
    kda_status s = check_prefill(q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, B, T, H, d_k, d_v, dtype,
                                 d_out_dtype, d_out, d_final_state, kda::kGateChannel);
    if (s != KDA_OK) return s;
    if (T > 0 && (!dq || !dk || !dv || !dlog_alpha || !dbeta)) return KDA_ERR_INVALID_ARG;
    const void *outs[] = {dq, dk, dv, dlog_alpha, dbeta, d_init_state};
    for (const void *p : outs)
        if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (chunk < 0) return KDA_ERR_INVALID_ARG;   // 0: every state stored, no recompute
    if (chunk > 256) return KDA_ERR_UNSUPPORTED;
    const int N = cu_seqlens ? num_seqs : B;
    const int64_t total = cu_seqlens ? (int64_t)T : (int64_t)B * T;
    const size_t need = kda::bwd_workspace_bytes(N, H, total, d_k, d_v, chunk);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dtype == KDA_F32)
        e = d_out_dtype == KDA_F32
                ? kda::launch_bwd<float, float>(d_k, d_v, q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, B,
                                                T, H, chunk, d_out, d_final_state, dq, dk, dv, dlog_alpha, dbeta,
                                                d_init_state, workspace, st)
                : kda::launch_bwd<float, __nv_bfloat16>(d_k, d_v, q, k, v, log_alpha, beta, init_state, cu_seqlens,
                                                        num_seqs, B, T, H, chunk, d_out, d_final_state, dq, dk, dv,
                                                        dlog_alpha, dbeta, d_init_state, workspace, st);
    else
        e = d_out_dtype == KDA_F32
                ? kda::launch_bwd<__nv_bfloat16, float>(d_k, d_v, q, k, v, log_alpha, beta, init_state, cu_seqlens,
                                                        num_seqs, B, T, H, chunk, d_out, d_final_state, dq, dk, dv,
                                                        dlog_alpha, dbeta, d_init_state, workspace, st)
                : kda::launch_bwd<__nv_bfloat16, __nv_bfloat16>(d_k, d_v, q, k, v, log_alpha, beta, init_state,
                                                                cu_seqlens, num_seqs, B, T, H, chunk, d_out,
                                                                d_final_state, dq, dk, dv, dlog_alpha, dbeta,
                                                                d_init_state, workspace, st);
    return from_cuda(e);
}

}  // extern "C"
