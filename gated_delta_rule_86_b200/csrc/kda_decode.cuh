// kda_decode.cuh -- single-token KDA decode step, fp32 state updated in place.
//
// One step of the recurrence of "Hybrid Linear Attention Architectures:
// Breaking Through the Long-Context Engineering Bottleneck in LLMs" (section
// "Core Module Design", Stage 3) for every (batch, head):
//     S' = Diag(alpha) S,   u = beta (v - S'^T k),   S = S' + k u^T,   o = S^T q.
// The two reductions over d_k share one pass over S':  S^T q = S'^T q + u (k.q),
// so every state element is read from HBM once and written once, which is the
// memory-bound decode regime that section 1 of "Linear Attention + Sparse
// Attention: The Hybrid Architecture Trade-off for Large Models" describes.
//
// The gate is one log-decay per key channel (KDA) or, with GK = kGateHead, one per head (Gated
// DeltaNet; a null gate gives DeltaNet, alpha == 1).  With GK = kRawInputs the token inputs are
// the raw projections: q and k are L2-normalised here, alpha = sigmoid(g), beta = sigmoid(b).
//
// Mapping: one CTA of 256 threads per (b, h).  Warp w owns state rows
// [w*DK/8, (w+1)*DK/8); lane l owns columns [l*DV/32, (l+1)*DV/32), so a warp
// reads and writes whole 128/256/512-byte rows (fully coalesced 16-byte
// accesses for DV = 128).  The state slice lives in registers between the read
// and the write.  Loads of the state are issued before the token vectors are
// staged so that HBM latency overlaps the staging.
#pragma once

#include "kda_common.cuh"

namespace kda {

template <int N> struct FVec;
template <> struct FVec<4> { using T = float4; };
template <> struct FVec<2> { using T = float2; };

__device__ __forceinline__ void fvec_to_arr(const float4 &v, float *a) { a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w; }
__device__ __forceinline__ void fvec_to_arr(const float2 &v, float *a) { a[0] = v.x; a[1] = v.y; }
__device__ __forceinline__ float4 arr_to_fvec4(const float *a) { return make_float4(a[0], a[1], a[2], a[3]); }
__device__ __forceinline__ float2 arr_to_fvec2(const float *a) { return make_float2(a[0], a[1]); }

template <int DK, int DV, typename TIO, typename TOUT, int GK>
__global__ void __launch_bounds__(256, 2)
kda_decode_kernel(const TIO *__restrict__ q, const TIO *__restrict__ k, const TIO *__restrict__ v,
                  const TIO *__restrict__ log_alpha, const TIO *__restrict__ beta, float *__restrict__ state,
                  TOUT *__restrict__ out) {
    constexpr int RPW = DK / 8;   // state rows per warp
    constexpr int CPL = DV / 32;  // state columns per lane
    using VecT = typename FVec<CPL>::T;

    __shared__ float s_q[DK], s_k[DK], s_a[DK], s_v[DV], s_u[DV];
    __shared__ __align__(16) float s_red[2][8][DV];
    __shared__ float s_kq[8];
    __shared__ float s_beta;
    __shared__ float s_nrm[2][DK / 32];   // raw inputs: per-warp sums of q^2 and k^2

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t head = blockIdx.x;
    float *S = state + head * (size_t)(DK * DV);

    // 1. issue the state loads (streaming: the state is read once per step)
    float s[RPW][CPL];
#pragma unroll
    for (int m = 0; m < RPW; ++m) {
        const VecT x = __ldcs(reinterpret_cast<const VecT *>(S + (warp * RPW + m) * DV + lane * CPL));
        fvec_to_arr(x, s[m]);
    }

    // 2. stage the token vectors
    if (tid < DK) {
        const float qv = to_f32(q[head * DK + tid]), kv = to_f32(k[head * DK + tid]);
        s_q[tid] = qv;
        s_k[tid] = kv;
        s_a[tid] = expf(gate_log<GK>(log_alpha, head, DK, tid));
        if constexpr (GK == kRawInputs) {   // partial sums for the L2 norms of the raw q and k
            float sq = qv * qv, sk = kv * kv;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
            }
            if (lane == 0) {
                s_nrm[0][warp] = sq;
                s_nrm[1][warp] = sk;
            }
        }
    }
    if (tid >= 256 - DV) s_v[tid - (256 - DV)] = to_f32(v[head * DV + tid - (256 - DV)]);
    if (tid == 0) s_beta = beta_of<GK>(beta, head);
    __syncthreads();
    // 1 / L2 norms of q and k (1 unless the inputs are raw projections)
    float nq = 1.f, nk = 1.f;
    if constexpr (GK == kRawInputs) {
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int w = 0; w < DK / 32; ++w) {
            sq += s_nrm[0][w];
            sk += s_nrm[1][w];
        }
        nq = rsqrtf(sq + kNormEps);
        nk = rsqrtf(sk + kNormEps);
    }

    // 3. decay in registers and per-warp partial reductions over this warp's rows
    float pa[CPL], pb[CPL];
    float kq = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) pa[c] = pb[c] = 0.f;
#pragma unroll
    for (int m = 0; m < RPW; ++m) {
        const int row = warp * RPW + m;
        const float a = s_a[row], kk = s_k[row] * nk, qq = s_q[row] * nq;
        kq = fmaf(kk, qq, kq);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            s[m][c] *= a;
            pa[c] = fmaf(s[m][c], kk, pa[c]);
            pb[c] = fmaf(s[m][c], qq, pb[c]);
        }
    }
    if constexpr (CPL == 4) {
        *reinterpret_cast<float4 *>(&s_red[0][warp][lane * 4]) = arr_to_fvec4(pa);
        *reinterpret_cast<float4 *>(&s_red[1][warp][lane * 4]) = arr_to_fvec4(pb);
    } else {
        *reinterpret_cast<float2 *>(&s_red[0][warp][lane * 2]) = arr_to_fvec2(pa);
        *reinterpret_cast<float2 *>(&s_red[1][warp][lane * 2]) = arr_to_fvec2(pb);
    }
    if (lane == 0) s_kq[warp] = kq;
    __syncthreads();

    // 4. finish the reductions: one thread per value column
    if (tid < DV) {
        float a = 0.f, b = 0.f, kqs = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            a += s_red[0][w][tid];
            b += s_red[1][w][tid];
            kqs += s_kq[w];
        }
        const float u = s_beta * (s_v[tid] - a);
        s_u[tid] = u;
        out[head * DV + tid] = from_f32<TOUT>(fmaf(u, kqs, b));
    }
    __syncthreads();

    // 5. rank-1 write and store
    float u[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) u[c] = s_u[lane * CPL + c];
#pragma unroll
    for (int m = 0; m < RPW; ++m) {
        const float kk = s_k[warp * RPW + m] * nk;
#pragma unroll
        for (int c = 0; c < CPL; ++c) s[m][c] = fmaf(kk, u[c], s[m][c]);
        VecT x;
        if constexpr (CPL == 4) x = arr_to_fvec4(s[m]); else x = arr_to_fvec2(s[m]);
        __stcs(reinterpret_cast<VecT *>(S + (warp * RPW + m) * DV + lane * CPL), x);
    }
}

template <int DK, int DV, typename TIO, typename TOUT, int GK = kGateChannel>
cudaError_t launch_decode(const void *q, const void *k, const void *v, const void *la, const void *beta,
                          float *state, void *out, int B, int H, cudaStream_t stream) {
    const unsigned grid = static_cast<unsigned>(B) * static_cast<unsigned>(H);
    kda_decode_kernel<DK, DV, TIO, TOUT, GK><<<grid, 256, 0, stream>>>(
        static_cast<const TIO *>(q), static_cast<const TIO *>(k), static_cast<const TIO *>(v),
        static_cast<const TIO *>(la), static_cast<const TIO *>(beta), state, static_cast<TOUT *>(out));
    return cudaGetLastError();
}

}  // namespace kda
