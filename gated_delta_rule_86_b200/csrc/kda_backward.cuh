// kda_backward.cuh -- gradient of the KDA prefill (reverse mode), fp32 on CUDA cores.
//
// The forward operator is the token recurrence of "Hybrid Linear Attention Architectures: Breaking
// Through the Long-Context Engineering Bottleneck in LLMs" (section "Core Module Design", Stage 3),
// written per token as
//     S' = Diag(a) S_prev,  a = exp(log_alpha)      w = S'^T k      u = beta (v - w)
//     S  = S' + k u^T                                o = S^T q
// The pages train this layer (their implementation checklist asks for FP32 intermediates and
// gradient clipping; section 3 of "Linear Attention KDA Gating in a 3:1 Hybrid Architecture" asks
// for gradient checks when the chunk size is chosen) but print no backward pass, so the kernel
// evaluates the plain adjoint of that step.  Given dS (the gradient with respect to the state after
// the token) and do:
//     dS   += q do^T                dq = S do
//     du    = dS^T k                dk = dS u - beta S' du
//     dbeta = du . (v - w)          dv = beta du
//     dS'   = dS - beta k du^T      dlog_alpha = rowsum(dS' * S')
//     dS_prev = Diag(a) dS'
// The result equals the gradient of the chunked forward up to rounding, because the chunked
// forward equals the recurrence.
//
// Schedule.  One CTA per (sequence, head).  Thread (warp w, lane l) owns key rows
// [32 (w / NCG), +32) and value column 32 (w % NCG) + l of the d_k x d_v state and of its gradient,
// in fp32 registers, so every sum over d_v or d_k is a shuffle transpose-sum inside a warp plus a
// deterministic combine across warps in shared memory (no atomics: results are reproducible).
//   1. forward over the sequence, storing the state at the start of every chunk of C tokens
//      (the checkpoints, in the workspace);
//   2. chunks in reverse: the chunk's states are recomputed from its checkpoint into a per-CTA
//      scratch (one d_k x d_v state per token), then its tokens are visited in reverse.
// Token vectors move through shared memory 32 tokens at a time.  Each token costs three passes of
// the recurrence (checkpoint pass, recompute, reverse), all in fp32.
#pragma once

#include "kda_common.cuh"

namespace kda {

namespace bwd {

constexpr int kSub = 32;   // tokens per staged block

// Lane l ends with the warp-wide sum of value l (recursive halving, 31 shuffles for 32 values).
__device__ __forceinline__ float transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = upper ? v[i] : v[i + off];
            const float keep = upper ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

template <int DK, int DV> struct Smem {
    static constexpr int NRG = DK / 32, NCG = DV / 32;
    static constexpr int kQ = 0;                       // [kSub][DK]
    static constexpr int kK = kQ + kSub * DK;          // [kSub][DK]
    static constexpr int kA = kK + kSub * DK;          // [kSub][DK]  exp(log_alpha)
    static constexpr int kV = kA + kSub * DK;          // [kSub][DV]
    static constexpr int kDo = kV + kSub * DV;         // [kSub][DV]
    static constexpr int kB = kDo + kSub * DV;         // [kSub]
    static constexpr int kRedW = kB + kSub;            // [2][NRG][DV]
    static constexpr int kRedDu = kRedW + 2 * NRG * DV;   // [NRG][DV]
    static constexpr int kRedQ = kRedDu + NRG * DV;    // [NCG][DK]
    static constexpr int kRedK = kRedQ + NCG * DK;     // [NCG][DK]
    static constexpr int kRedG = kRedK + NCG * DK;     // [NCG][DK]
    static constexpr int kRedB = kRedG + NCG * DK;     // [NCG]
    static constexpr int kFloats = kRedB + NCG;
};

// Checkpoint slots of the sequence whose tokens start at t0: sequences never share one
// (floor(t0 / C) + n is at least the number of chunks of all earlier sequences, and the ranges of
// consecutive sequences do not overlap).
__host__ __device__ __forceinline__ int64_t ckpt_base(int64_t t0, int n, int C) { return t0 / C + n; }
inline int64_t ckpts_per_head(int64_t total_tokens, int N, int C) { return total_tokens / C + N + 1; }

}  // namespace bwd

template <int DK, int DV, typename TIO, typename TDO>
__global__ void __launch_bounds__(32 * (DK / 32) * (DV / 32))
kda_bwd_kernel(const TIO *__restrict__ q, const TIO *__restrict__ k, const TIO *__restrict__ v,
               const TIO *__restrict__ log_alpha, const TIO *__restrict__ beta, const float *init_state,
               const int32_t *__restrict__ cu, int T, int H, int C, const TDO *__restrict__ dout,
               const float *dfinal, float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
               float *__restrict__ dla, float *__restrict__ dbeta, float *dinit, float *ckpt, float *scratch,
               int64_t nck_head) {
    using SM = bwd::Smem<DK, DV>;
    constexpr int NRG = SM::NRG, NCG = SM::NCG, NT = 32 * NRG * NCG;
    constexpr int kSub = bwd::kSub;
    extern __shared__ float smf[];
    float *sq = smf + SM::kQ, *sk = smf + SM::kK, *sa = smf + SM::kA, *sv = smf + SM::kV, *sdo = smf + SM::kDo;
    float *sb = smf + SM::kB, *red_w = smf + SM::kRedW, *red_du = smf + SM::kRedDu, *red_q = smf + SM::kRedQ;
    float *red_k = smf + SM::kRedK, *red_g = smf + SM::kRedG, *red_b = smf + SM::kRedB;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rg = warp / NCG, cg = warp % NCG;
    const int j = cg * 32 + lane, r0 = rg * 32;
    const int pair = blockIdx.x, h = pair % H, n = pair / H;
    const int64_t t0 = cu ? (int64_t)cu[n] : (int64_t)n * T;
    const int64_t t1 = cu ? (int64_t)cu[n + 1] : t0 + T;
    const int L = static_cast<int>(t1 - t0);
    const int nck = (L + C - 1) / C;
    const size_t kv = (size_t)DK * DV;
    float *my_ck = ckpt + ((size_t)h * nck_head + bwd::ckpt_base(t0, n, C)) * kv;
    float *my_scr = scratch + (size_t)pair * C * kv;
    const size_t sbase = ((size_t)n * H + h) * kv;
    auto el = [&](int m) { return (size_t)(r0 + m) * DV + j; };   // this thread's element of row r0 + m

    // stage tokens [ts, ts + nb) of the sequence (need_q: also q and do)
    auto stage = [&](int ts, int nb, bool need_q) {
        __syncthreads();   // every thread is done with the previous block
        for (int idx = tid; idx < nb * DK; idx += NT) {
            const int tk = idx / DK, c = idx - tk * DK;
            const size_t row = (size_t)(t0 + ts + tk) * H + h;
            sk[tk * DK + c] = to_f32(k[row * DK + c]);
            sa[tk * DK + c] = expf(to_f32(log_alpha[row * DK + c]));
            if (need_q) sq[tk * DK + c] = to_f32(q[row * DK + c]);
        }
        for (int idx = tid; idx < nb * DV; idx += NT) {
            const int tk = idx / DV, c = idx - tk * DV;
            const size_t row = (size_t)(t0 + ts + tk) * H + h;
            sv[tk * DV + c] = to_f32(v[row * DV + c]);
            if (need_q) sdo[tk * DV + c] = to_f32(dout[row * DV + c]);
        }
        for (int tk = tid; tk < nb; tk += NT) sb[tk] = to_f32(beta[(size_t)(t0 + ts + tk) * H + h]);
        __syncthreads();
    };
    // one forward step of the staged token i on the state S (one barrier; red_w is double-buffered)
    int wbuf = 0;
    auto forward_step = [&](float (&S)[32], int i) {
        float pw = 0.f;
#pragma unroll
        for (int m = 0; m < 32; ++m) {
            S[m] *= sa[i * DK + r0 + m];
            pw = fmaf(S[m], sk[i * DK + r0 + m], pw);
        }
        red_w[(wbuf * NRG + rg) * DV + j] = pw;
        __syncthreads();
        float w = 0.f;
#pragma unroll
        for (int g = 0; g < NRG; ++g) w += red_w[(wbuf * NRG + g) * DV + j];
        wbuf ^= 1;
        const float u = sb[i] * (sv[i * DV + j] - w);
#pragma unroll
        for (int m = 0; m < 32; ++m) S[m] = fmaf(sk[i * DK + r0 + m], u, S[m]);
    };

    // ---- 1. forward with a checkpoint at the start of every chunk ----
    {
        float S[32];
#pragma unroll
        for (int m = 0; m < 32; ++m) S[m] = init_state ? init_state[sbase + el(m)] : 0.f;
        for (int c = 0; c < nck; ++c) {
#pragma unroll
            for (int m = 0; m < 32; ++m) my_ck[(size_t)c * kv + el(m)] = S[m];
            if (c == nck - 1) break;   // the last chunk's tokens are recomputed in step 2
            for (int ts = c * C; ts < (c + 1) * C; ts += kSub) {
                const int nb = min(kSub, (c + 1) * C - ts);
                stage(ts, nb, false);
                for (int i = 0; i < nb; ++i) forward_step(S, i);
            }
        }
    }

    // ---- 2. chunks in reverse ----
    float dS[32];
#pragma unroll
    for (int m = 0; m < 32; ++m) dS[m] = dfinal ? dfinal[sbase + el(m)] : 0.f;
    for (int c = nck - 1; c >= 0; --c) {
        const int cs = c * C, ce = min(L, cs + C);
        // recompute: the state before every token of the chunk, into the scratch
        {
            float S[32];
#pragma unroll
            for (int m = 0; m < 32; ++m) S[m] = my_ck[(size_t)c * kv + el(m)];
            for (int ts = cs; ts < ce; ts += kSub) {
                const int nb = min(kSub, ce - ts);
                stage(ts, nb, false);
                for (int i = 0; i < nb; ++i) {
#pragma unroll
                    for (int m = 0; m < 32; ++m) my_scr[(size_t)(ts - cs + i) * kv + el(m)] = S[m];
                    forward_step(S, i);
                }
            }
        }
        // reverse over the chunk's tokens, in staged blocks from the end
        const int nblk = (ce - cs + kSub - 1) / kSub;
        for (int bi = nblk - 1; bi >= 0; --bi) {
            const int ts = cs + bi * kSub, nb = min(kSub, ce - ts);
            stage(ts, nb, true);
            for (int i = nb - 1; i >= 0; --i) {
                const size_t trow = (size_t)(t0 + ts + i) * H + h;
                // S' = Diag(a) S_prev and w = S'^T k
                float Sp[32];
                float pw = 0.f;
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    Sp[m] = sa[i * DK + r0 + m] * my_scr[(size_t)(ts - cs + i) * kv + el(m)];
                    pw = fmaf(Sp[m], sk[i * DK + r0 + m], pw);
                }
                red_w[(wbuf * NRG + rg) * DV + j] = pw;
                __syncthreads();
                float w = 0.f;
#pragma unroll
                for (int g = 0; g < NRG; ++g) w += red_w[(wbuf * NRG + g) * DV + j];
                wbuf ^= 1;
                const float bt = sb[i], vj = sv[i * DV + j], doj = sdo[i * DV + j];
                const float u = bt * (vj - w);
                // o = S^T q: dS += q do^T, dq = S do (S = S' + k u^T)
                float x[32];
                float pdu = 0.f;
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    const float km = sk[i * DK + r0 + m];
                    dS[m] = fmaf(sq[i * DK + r0 + m], doj, dS[m]);
                    x[m] = fmaf(km, u, Sp[m]) * doj;
                    pdu = fmaf(dS[m], km, pdu);   // du = dS^T k
                }
                red_q[cg * DK + r0 + lane] = bwd::transpose_sum32(x, lane);
                red_du[rg * DV + j] = pdu;
                __syncthreads();
                float du = 0.f;
#pragma unroll
                for (int g = 0; g < NRG; ++g) du += red_du[g * DV + j];
                if (rg == 0) {
                    dv[trow * DV + j] = bt * du;
                    float db = du * (vj - w);
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) db += __shfl_xor_sync(0xffffffffu, db, o);
                    if (lane == 0) red_b[cg] = db;
                }
                // dk = dS u - beta S' du;  dS' = dS - beta k du^T;  dlog_alpha = rowsum(dS' * S');  dS = a dS'
#pragma unroll
                for (int m = 0; m < 32; ++m) x[m] = dS[m] * u - bt * Sp[m] * du;
                red_k[cg * DK + r0 + lane] = bwd::transpose_sum32(x, lane);
#pragma unroll
                for (int m = 0; m < 32; ++m) {
                    dS[m] = fmaf(-bt * sk[i * DK + r0 + m], du, dS[m]);
                    x[m] = dS[m] * Sp[m];
                    dS[m] *= sa[i * DK + r0 + m];
                }
                red_g[cg * DK + r0 + lane] = bwd::transpose_sum32(x, lane);
                __syncthreads();
                if (tid < DK) {
                    float aq = 0.f, ak = 0.f, ag = 0.f;
#pragma unroll
                    for (int g = 0; g < NCG; ++g) {
                        aq += red_q[g * DK + tid];
                        ak += red_k[g * DK + tid];
                        ag += red_g[g * DK + tid];
                    }
                    dq[trow * DK + tid] = aq;
                    dk[trow * DK + tid] = ak;
                    dla[trow * DK + tid] = ag;
                }
                if (tid == DK % NT) {
                    float ab = 0.f;
#pragma unroll
                    for (int g = 0; g < NCG; ++g) ab += red_b[g];
                    dbeta[trow] = ab;
                }
            }
        }
    }
    if (dinit) {
#pragma unroll
        for (int m = 0; m < 32; ++m) dinit[sbase + el(m)] = dS[m];
    }
}

// Workspace of the backward: the checkpoints (one d_k x d_v state per chunk of every sequence and
// head) and one chunk's per-token states for every (sequence, head) pair.
inline size_t bwd_workspace_bytes(int64_t N, int64_t H, int64_t total_tokens, int DK, int DV, int C) {
    const size_t kv = (size_t)DK * DV * sizeof(float);
    return (size_t)H * bwd::ckpts_per_head(total_tokens, (int)N, C) * kv + (size_t)N * H * C * kv;
}

template <int DK, int DV, typename TIO, typename TDO>
cudaError_t launch_bwd_dk_dv(const void *q, const void *k, const void *v, const void *la, const void *beta,
                             const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H, int C,
                             const void *dout, const float *dfinal, float *dq, float *dk, float *dv, float *dla,
                             float *dbeta, float *dinit, void *workspace, cudaStream_t stream) {
    using SM = bwd::Smem<DK, DV>;
    auto kern = kda_bwd_kernel<DK, DV, TIO, TDO>;
    const int smem = SM::kFloats * static_cast<int>(sizeof(float));
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int N = cu ? num_seqs : B;
    const int64_t total = cu ? (int64_t)T : (int64_t)B * T;   // with cu_seqlens, T is the packed length
    const int64_t nck_head = bwd::ckpts_per_head(total, N, C);
    float *ck = static_cast<float *>(workspace);
    float *scr = ck + (size_t)H * nck_head * DK * DV;
    const unsigned grid = static_cast<unsigned>(N) * H;
    if (grid == 0) return cudaSuccess;
    kern<<<grid, 32 * (DK / 32) * (DV / 32), smem, stream>>>(
        static_cast<const TIO *>(q), static_cast<const TIO *>(k), static_cast<const TIO *>(v),
        static_cast<const TIO *>(la), static_cast<const TIO *>(beta), init_state, cu, T, H, C,
        static_cast<const TDO *>(dout), dfinal, dq, dk, dv, dla, dbeta, dinit, ck, scr, nck_head);
    return cudaGetLastError();
}

template <typename TIO, typename TDO>
cudaError_t launch_bwd(int DK, int DV, const void *q, const void *k, const void *v, const void *la, const void *beta,
                       const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H, int C,
                       const void *dout, const float *dfinal, float *dq, float *dk, float *dv, float *dla,
                       float *dbeta, float *dinit, void *workspace, cudaStream_t stream) {
#define KDA_BWD_CASE(A, Bv)                                                                                 \
    if (DK == A && DV == Bv)                                                                                \
        return launch_bwd_dk_dv<A, Bv, TIO, TDO>(q, k, v, la, beta, init_state, cu, num_seqs, B, T, H, C, dout, \
                                                 dfinal, dq, dk, dv, dla, dbeta, dinit, workspace, stream);
    KDA_BWD_CASE(64, 64)
    KDA_BWD_CASE(64, 128)
    KDA_BWD_CASE(128, 64)
    KDA_BWD_CASE(128, 128)
#undef KDA_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace kda
