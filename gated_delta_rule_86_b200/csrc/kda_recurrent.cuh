// kda_recurrent.cuh -- token-by-token KDA prefill on CUDA cores, fp32 state.
//
// Evaluates the recurrence of "Hybrid Linear Attention Architectures: Breaking
// Through the Long-Context Engineering Bottleneck in LLMs" (section "Core
// Module Design", Stage 3) one token at a time, with the state slice held in
// fp32 registers for the whole sequence.  This is the RNN mode that section 3
// of "Linear Attention KDA Gating in a 3:1 Hybrid Architecture" contrasts with
// the chunked algorithm; here it serves as the fp32-accurate prefill (fp32 I/O)
// and as the token-by-token point of comparison for the chunked kernel.
//
// The gate is one log-decay per key channel (KDA) or, with GK = kGateHead, one per head and token
// (Gated DeltaNet; a null gate gives DeltaNet, alpha == 1).
//
// Mapping: one CTA of 128 threads per (sequence, head, 32-column slice of d_v).
// Lane l owns value column l of the slice; warp w owns key rows
// [w*DK/4, (w+1)*DK/4), so each thread keeps DK/4 state values in registers.
// Per token: decay + partial reductions over the thread's rows, one
// __syncthreads, a 4-way combine through shared memory, then the rank-1 write.
// Token vectors go through a 3-deep shared-memory ring filled one token ahead
// from registers that were loaded two tokens ahead, so global-load latency is
// hidden behind the previous token's arithmetic.
#pragma once

#include "kda_common.cuh"

namespace kda {

// Sequence index processed at position `p` of a longest-first order over
// packed sequences (ties broken by index).  O(num_seqs^2 / blockDim) work; the
// caller only uses it for modest num_seqs and falls back to p otherwise.
__device__ __forceinline__ int longest_first_seq(const int32_t *cu, int num_seqs, int p, int *s_slot) {
    if (threadIdx.x == 0) *s_slot = p;
    __syncthreads();
    for (int n = threadIdx.x; n < num_seqs; n += blockDim.x) {
        const int ln = cu[n + 1] - cu[n];
        int rank = 0;
        for (int m = 0; m < num_seqs; ++m) {
            const int lm = cu[m + 1] - cu[m];
            rank += (lm > ln) || (lm == ln && m < n);
        }
        if (rank == p) *s_slot = n;
    }
    __syncthreads();
    const int r = *s_slot;
    __syncthreads();
    return r;
}

constexpr int kLongestFirstMaxSeqs = 1024;

template <int DK, typename TIO, typename TOUT, int GK>
__global__ void __launch_bounds__(128)
kda_recurrent_kernel(const TIO *__restrict__ q, const TIO *__restrict__ k, const TIO *__restrict__ v,
                     const TIO *__restrict__ log_alpha, const TIO *__restrict__ beta,
                     const float *init_state, const int32_t *__restrict__ cu_seqlens, int num_seqs, int T,
                     int H, int DV, TOUT *__restrict__ out, float *final_state) {
    constexpr int RPW = DK / 4;  // rows per warp
    __shared__ float s_q[3][DK], s_k[3][DK], s_a[3][DK], s_v[3][32], s_b[3];
    __shared__ float s_red[2][2][4][32];
    __shared__ float s_kq[2][4];
    __shared__ int s_slot;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nslices = DV / 32;
    const int slice = blockIdx.x % nslices;
    const int pair = blockIdx.x / nslices;  // (sequence position, head)
    const int h = pair % H;
    int n = pair / H;
    int64_t t0, t1;
    if (cu_seqlens) {
        if (num_seqs <= kLongestFirstMaxSeqs) n = longest_first_seq(cu_seqlens, num_seqs, n, &s_slot);
        t0 = cu_seqlens[n];
        t1 = cu_seqlens[n + 1];
    } else {
        t0 = (int64_t)n * T;  // flattened [B*T] token index of this batch row
        t1 = t0 + T;
    }
    const int L = static_cast<int>(t1 - t0);
    const int col = slice * 32 + lane;

    float s[RPW];
    const size_t sbase = ((size_t)n * H + h) * DK * DV;
#pragma unroll
    for (int m = 0; m < RPW; ++m)
        s[m] = init_state ? init_state[sbase + (size_t)(warp * RPW + m) * DV + col] : 0.f;

    // register prefetch of one token's vectors (thread tid < DK: q, k, log_alpha; tid < 32: v; tid == 0: beta)
    float rq = 0.f, rk = 0.f, ra = 0.f, rv = 0.f, rb = 0.f;
    auto fetch = [&](int t) {
        if (t >= L) return;
        const size_t row = (size_t)(t0 + t) * H + h;
        if (tid < DK) {
            rq = to_f32(q[row * DK + tid]);
            rk = to_f32(k[row * DK + tid]);
            ra = gate_log<GK>(log_alpha, row, DK, tid);
        }
        if (tid < 32) rv = to_f32(v[row * DV + slice * 32 + tid]);
        if (tid == 0) rb = to_f32(beta[row]);
    };
    auto stage = [&](int t) {
        if (t >= L) return;
        const int b = t % 3;
        if (tid < DK) {
            s_q[b][tid] = rq;
            s_k[b][tid] = rk;
            s_a[b][tid] = expf(ra);
        }
        if (tid < 32) s_v[b][tid] = rv;
        if (tid == 0) s_b[b] = rb;
    };

    fetch(0);
    stage(0);
    fetch(1);
    __syncthreads();

    for (int t = 0; t < L; ++t) {
        const int b = t % 3, r = t & 1;
        // (1) decay and partial reductions over this warp's rows
        float pa = 0.f, pb = 0.f, kq = 0.f;
#pragma unroll
        for (int m = 0; m < RPW; ++m) {
            const int row = warp * RPW + m;
            const float kk = s_k[b][row], qq = s_q[b][row];
            s[m] *= s_a[b][row];
            pa = fmaf(s[m], kk, pa);
            pb = fmaf(s[m], qq, pb);
            kq = fmaf(kk, qq, kq);
        }
        s_red[r][0][warp][lane] = pa;
        s_red[r][1][warp][lane] = pb;
        if (lane == 0) s_kq[r][warp] = kq;
        // (2) stage token t+1 (loaded last iteration), load token t+2
        stage(t + 1);
        fetch(t + 2);
        __syncthreads();
        // (3) combine, output, rank-1 write
        float a = 0.f, bq = 0.f, kqs = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            a += s_red[r][0][w][lane];
            bq += s_red[r][1][w][lane];
            kqs += s_kq[r][w];
        }
        const float u = s_b[b] * (s_v[b][lane] - a);
        if (warp == 0) out[((size_t)(t0 + t) * H + h) * DV + col] = from_f32<TOUT>(fmaf(u, kqs, bq));
#pragma unroll
        for (int m = 0; m < RPW; ++m) s[m] = fmaf(s_k[b][warp * RPW + m], u, s[m]);
    }

    if (final_state) {
#pragma unroll
        for (int m = 0; m < RPW; ++m) final_state[sbase + (size_t)(warp * RPW + m) * DV + col] = s[m];
    }
}

template <int DK, typename TIO, typename TOUT, int GK = kGateChannel>
cudaError_t launch_recurrent(const void *q, const void *k, const void *v, const void *la, const void *beta,
                             const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H, int DV,
                             void *out, float *final_state, cudaStream_t stream) {
    const int N = cu ? num_seqs : B;
    const unsigned grid = static_cast<unsigned>(N) * H * (DV / 32);
    kda_recurrent_kernel<DK, TIO, TOUT, GK><<<grid, 128, 0, stream>>>(
        static_cast<const TIO *>(q), static_cast<const TIO *>(k), static_cast<const TIO *>(v),
        static_cast<const TIO *>(la), static_cast<const TIO *>(beta), init_state, cu, num_seqs, T, H, DV,
        static_cast<TOUT *>(out), final_state);
    return cudaGetLastError();
}

}  // namespace kda
