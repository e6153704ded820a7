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
// Schedule.  One cluster of d_v / 32 CTAs per (sequence, head); CTA s of the cluster owns value
// columns [32 s, 32 s + 32) of the d_k x d_v state and of its gradient (the columns evolve
// independently).  Thread (warp w, lane l) owns key rows [R w, R w + R) (R = kRows) and column
// 32 s + l, in fp32 registers, so every sum over d_k is a combine of the warps' partials in shared
// memory, and every sum over d_v is a shuffle transpose-sum inside a warp (the CTA's 32 columns) plus
// a combine of the cluster's slices through distributed shared memory, once per block of 32 tokens.  Both
// combines run in a fixed order (no atomics: results are reproducible).
//   1. forward over the sequence, storing the state at the start of every chunk of C tokens
//      (the checkpoints, in the workspace);
//   2. chunks in reverse: the chunk's states are recomputed from its checkpoint into a per-pair
//      scratch (one d_k x d_v state per token), then its tokens are visited in reverse.
// With C = 0 ("every state") step 1 stores the state before every token instead and step 2 reads
// those (no recompute; the workspace then holds one state per token and head); the states, and so
// the results, are bitwise those of the checkpointed schedule.
// Token vectors move through shared memory 32 tokens at a time.  Each token costs three passes of
// the recurrence (checkpoint pass, recompute, reverse), all in fp32.
#pragma once

#include "kda_common.cuh"

namespace kda {

namespace bwd {

constexpr int kSub = 32;   // tokens per staged block
#ifndef KDA_BWD_ROWS
#define KDA_BWD_ROWS 8
#endif
constexpr int kRows = KDA_BWD_ROWS;   // key rows per thread: d_k / kRows warps per CTA
static_assert(kRows == 8 || kRows == 16 || kRows == 32, "rows per thread");

// Sum over the warp's 32 lanes of each of the kRows values v[m]: lane l ends with the sum of value
// l % kRows (recursive halving inside groups of kRows lanes, then adds across the groups:
// kRows - 1 + log2(32 / kRows) shuffles).
__device__ __forceinline__ float transpose_sum_rows(float (&v)[kRows], int lane) {
#pragma unroll
    for (int off = kRows / 2; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = upper ? v[i] : v[i + off];
            const float keep = upper ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
#pragma unroll
    for (int off = kRows; off < 32; off <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    return v[0];
}

template <int DK, int DV> struct Smem {
    static constexpr int NRG = DK / kRows, NCS = DV / 32;   // warps per CTA, CTAs per cluster
    static constexpr int kQ = 0;                       // [kSub][DK]
    static constexpr int kK = kQ + kSub * DK;          // [kSub][DK]
    static constexpr int kA = kK + kSub * DK;          // [kSub][DK]  exp(log_alpha)
    static constexpr int kV = kA + kSub * DK;          // [kSub][32]  this CTA's value columns
    static constexpr int kDo = kV + kSub * 32;         // [kSub][32]
    static constexpr int kB = kDo + kSub * 32;         // [kSub]
    static constexpr int kRedW = kB + kSub;            // [2][NRG][32]
    static constexpr int kRedDu = kRedW + 2 * NRG * 32;   // [NRG][32]
    // this slice's partial sums over its 32 columns, double-buffered by block: dq, dk, dlog_alpha
    // ([3][kSub][DK]) and dbeta ([kSub])
    static constexpr int kPart = kRedDu + NRG * 32;
    static constexpr int kPartFloats = 3 * kSub * DK + kSub;
    static constexpr int kFloats = kPart + 2 * kPartFloats;
};

// Checkpoint slots of the sequence whose tokens start at t0: sequences never share one
// (floor(t0 / C) + n is at least the number of chunks of all earlier sequences, and the ranges of
// consecutive sequences do not overlap).
__host__ __device__ __forceinline__ int64_t ckpt_base(int64_t t0, int n, int C) { return t0 / C + n; }
inline int64_t ckpts_per_head(int64_t total_tokens, int N, int C) { return total_tokens / C + N + 1; }

}  // namespace bwd

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster: arrive (release), then wait (acquire).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// fp32 load from the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ float ld_dsmem(const float *local, uint32_t rank) {
    uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local)), ra;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

template <int DK, int DV, typename TIO, typename TDO>
__global__ void __launch_bounds__(32 * (DK / bwd::kRows))
kda_bwd_kernel(const TIO *__restrict__ q, const TIO *__restrict__ k, const TIO *__restrict__ v,
               const TIO *__restrict__ log_alpha, const TIO *__restrict__ beta, const float *init_state,
               const int32_t *__restrict__ cu, int T, int H, int C, const TDO *__restrict__ dout,
               const float *dfinal, float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
               float *__restrict__ dla, float *__restrict__ dbeta, float *dinit, float *ckpt, float *scratch,
               int64_t nck_head) {
    using SM = bwd::Smem<DK, DV>;
    constexpr int NRG = SM::NRG, NCS = SM::NCS, NT = 32 * NRG;
    constexpr int kSub = bwd::kSub, R = bwd::kRows;
    extern __shared__ float smf[];
    float *sq = smf + SM::kQ, *sk = smf + SM::kK, *sa = smf + SM::kA, *sv = smf + SM::kV, *sdo = smf + SM::kDo;
    float *sb = smf + SM::kB, *red_w = smf + SM::kRedW, *red_du = smf + SM::kRedDu, *part = smf + SM::kPart;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rg = warp, r0 = rg * R;
    const int cs = static_cast<int>(cluster_ctarank());   // == blockIdx.x % NCS
    const int j = cs * 32 + lane;
    const int pair = blockIdx.x / NCS, h = pair % H, n = pair / H;
    const int64_t t0 = cu ? (int64_t)cu[n] : (int64_t)n * T;
    const int64_t t1 = cu ? (int64_t)cu[n + 1] : t0 + T;
    const int L = static_cast<int>(t1 - t0);
    const bool every = C == 0;   // the state before every token is stored in step 1: no recompute
    const int Ce = every ? (L > 0 ? L : 1) : C;
    const int nck = (L + Ce - 1) / Ce;
    const size_t kv = (size_t)DK * DV;
    float *my_ck = every ? nullptr : ckpt + ((size_t)h * nck_head + bwd::ckpt_base(t0, n, C)) * kv;
    // step 2's per-token states: the per-pair scratch of one chunk, or (every) this pair's tokens in
    // the workspace's [H][total tokens] states
    float *my_scr = every ? scratch + ((size_t)h * nck_head + t0) * kv : scratch + (size_t)pair * C * kv;
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
        for (int idx = tid; idx < nb * 32; idx += NT) {
            const int tk = idx >> 5, c = idx & 31;
            const size_t row = (size_t)(t0 + ts + tk) * H + h;
            sv[tk * 32 + c] = to_f32(v[row * DV + cs * 32 + c]);
            if (need_q) sdo[tk * 32 + c] = to_f32(dout[row * DV + cs * 32 + c]);
        }
        for (int tk = tid; tk < nb; tk += NT) sb[tk] = to_f32(beta[(size_t)(t0 + ts + tk) * H + h]);
        __syncthreads();
    };
    // this thread's R key rows of a staged token vector (16-byte shared-memory loads, the same
    // address across the warp)
    auto rows = [&](const float *base, float (&o)[R]) {
        const float4 *p4 = reinterpret_cast<const float4 *>(base + r0);
#pragma unroll
        for (int m4 = 0; m4 < R / 4; ++m4) {
            const float4 f = p4[m4];
            o[4 * m4] = f.x;
            o[4 * m4 + 1] = f.y;
            o[4 * m4 + 2] = f.z;
            o[4 * m4 + 3] = f.w;
        }
    };
    // one forward step of the staged token i on the state S (one barrier; red_w is double-buffered)
    int wbuf = 0;
    auto forward_step = [&](float (&S)[R], int i) {
        float ka[R], aa[R];
        rows(sk + i * DK, ka);
        rows(sa + i * DK, aa);
        float pw4[4] = {0.f, 0.f, 0.f, 0.f};   // four interleaved partial sums over the 32 rows
#pragma unroll
        for (int m = 0; m < R; ++m) {
            S[m] *= aa[m];
            pw4[m & 3] = fmaf(S[m], ka[m], pw4[m & 3]);
        }
        const float pw = (pw4[0] + pw4[1]) + (pw4[2] + pw4[3]);
        red_w[(wbuf * NRG + rg) * 32 + lane] = pw;
        __syncthreads();
        float w = 0.f;
#pragma unroll
        for (int g = 0; g < NRG; ++g) w += red_w[(wbuf * NRG + g) * 32 + lane];
        wbuf ^= 1;
        const float u = sb[i] * (sv[i * 32 + lane] - w);
#pragma unroll
        for (int m = 0; m < R; ++m) S[m] = fmaf(ka[m], u, S[m]);
    };

    // ---- 1. forward with a checkpoint at the start of every chunk (every: before every token) ----
    if (every) {
        float S[R];
#pragma unroll
        for (int m = 0; m < R; ++m) S[m] = init_state ? init_state[sbase + el(m)] : 0.f;
        for (int ts = 0; ts < L; ts += kSub) {
            const int nb = min(kSub, L - ts);
            stage(ts, nb, false);
            for (int i = 0; i < nb; ++i) {
#pragma unroll
                for (int m = 0; m < R; ++m) my_scr[(size_t)(ts + i) * kv + el(m)] = S[m];
                if (ts + i + 1 < L) forward_step(S, i);
            }
        }
    } else {
        float S[R];
#pragma unroll
        for (int m = 0; m < R; ++m) S[m] = init_state ? init_state[sbase + el(m)] : 0.f;
        for (int c = 0; c < nck; ++c) {
#pragma unroll
            for (int m = 0; m < R; ++m) my_ck[(size_t)c * kv + el(m)] = S[m];
            if (c == nck - 1) break;   // the last chunk's tokens are recomputed in step 2
            for (int ts = c * C; ts < (c + 1) * C; ts += kSub) {
                const int nb = min(kSub, (c + 1) * C - ts);
                stage(ts, nb, false);
                for (int i = 0; i < nb; ++i) forward_step(S, i);
            }
        }
    }

    // ---- 2. chunks in reverse ----
    float dS[R];
#pragma unroll
    for (int m = 0; m < R; ++m) dS[m] = dfinal ? dfinal[sbase + el(m)] : 0.f;
    int blk = 0;   // reverse blocks so far (selects the partial-sum buffer)
    for (int c = nck - 1; c >= 0; --c) {
        const int cs0 = c * Ce, ce = min(L, cs0 + Ce);
        // recompute: the state before every token of the chunk, into the scratch
        if (!every) {
            float S[R];
#pragma unroll
            for (int m = 0; m < R; ++m) S[m] = my_ck[(size_t)c * kv + el(m)];
            for (int ts = cs0; ts < ce; ts += kSub) {
                const int nb = min(kSub, ce - ts);
                stage(ts, nb, false);
                for (int i = 0; i < nb; ++i) {
#pragma unroll
                    for (int m = 0; m < R; ++m) my_scr[(size_t)(ts - cs0 + i) * kv + el(m)] = S[m];
                    forward_step(S, i);
                }
            }
        }
        // reverse over the chunk's tokens, in staged blocks from the end
        const int nblk = (ce - cs0 + kSub - 1) / kSub;
        for (int bi = nblk - 1; bi >= 0; --bi, ++blk) {
            const int ts = cs0 + bi * kSub, nb = min(kSub, ce - ts);
            float *pq = part + (blk & 1) * SM::kPartFloats, *pk = pq + kSub * DK, *pg = pk + kSub * DK;
            float *pb = pg + kSub * DK;
            stage(ts, nb, true);
            // the recomputed state before token i, loaded one token ahead of its use
            float Sn[R];
#pragma unroll
            for (int m = 0; m < R; ++m) Sn[m] = my_scr[(size_t)(ts - cs0 + nb - 1) * kv + el(m)];
            for (int i = nb - 1; i >= 0; --i) {
                float ka[R], aa[R];
                rows(sk + i * DK, ka);
                rows(sa + i * DK, aa);
                // S' = Diag(a) S_prev and w = S'^T k
                float Sp[R];
                float pw4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < R; ++m) {
                    Sp[m] = aa[m] * Sn[m];
                    pw4[m & 3] = fmaf(Sp[m], ka[m], pw4[m & 3]);
                }
                if (i > 0) {
#pragma unroll
                    for (int m = 0; m < R; ++m) Sn[m] = my_scr[(size_t)(ts - cs0 + i - 1) * kv + el(m)];
                }
                const float pw = (pw4[0] + pw4[1]) + (pw4[2] + pw4[3]);
                red_w[(wbuf * NRG + rg) * 32 + lane] = pw;
                __syncthreads();
                float w = 0.f;
#pragma unroll
                for (int g = 0; g < NRG; ++g) w += red_w[(wbuf * NRG + g) * 32 + lane];
                wbuf ^= 1;
                const float bt = sb[i], vj = sv[i * 32 + lane], doj = sdo[i * 32 + lane];
                const float u = bt * (vj - w);
                // o = S^T q: dS += q do^T, dq = S do (S = S' + k u^T)
                float x[R];
                {
                    float qa[R];
                    rows(sq + i * DK, qa);
                    float pdu4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int m = 0; m < R; ++m) {
                        dS[m] = fmaf(qa[m], doj, dS[m]);
                        x[m] = fmaf(ka[m], u, Sp[m]) * doj;
                        pdu4[m & 3] = fmaf(dS[m], ka[m], pdu4[m & 3]);   // du = dS^T k
                    }
                    red_du[rg * 32 + lane] = (pdu4[0] + pdu4[1]) + (pdu4[2] + pdu4[3]);
                }
                {
                    const float t = bwd::transpose_sum_rows(x, lane);
                    if (lane < R) pq[i * DK + r0 + lane] = t;
                }
                __syncthreads();
                float du = 0.f;
#pragma unroll
                for (int g = 0; g < NRG; ++g) du += red_du[g * 32 + lane];
                if (rg == 0) {
                    dv[((size_t)(t0 + ts + i) * H + h) * DV + j] = bt * du;
                    float db = du * (vj - w);
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) db += __shfl_xor_sync(0xffffffffu, db, o);
                    if (lane == 0) pb[i] = db;
                }
                // dk = dS u - beta S' du;  dS' = dS - beta k du^T;  dlog_alpha = rowsum(dS' * S');  dS = a dS'
#pragma unroll
                for (int m = 0; m < R; ++m) x[m] = dS[m] * u - bt * Sp[m] * du;
                {
                    const float t = bwd::transpose_sum_rows(x, lane);
                    if (lane < R) pk[i * DK + r0 + lane] = t;
                }
#pragma unroll
                for (int m = 0; m < R; ++m) {
                    dS[m] = fmaf(-bt * ka[m], du, dS[m]);
                    x[m] = dS[m] * Sp[m];
                    dS[m] *= aa[m];
                }
                {
                    const float t = bwd::transpose_sum_rows(x, lane);
                    if (lane < R) pg[i * DK + r0 + lane] = t;
                }
            }
            // the block's sums over d_v: every slice's partials are complete (cluster barrier), then
            // CTA s combines the elements e = s NT + tid, + NCS NT, ... over the slices in order 0, 1, ...
            // (the buffer is rewritten two blocks later, after every CTA has passed the next barrier)
            cluster_sync();
            for (int e = cs * NT + tid; e < nb * DK; e += NCS * NT) {
                const int i = e / DK, r = e - i * DK;
                float aq = 0.f, ak = 0.f, ag = 0.f;
#pragma unroll
                for (int g = 0; g < NCS; ++g) {
                    aq += ld_dsmem(pq + i * DK + r, g);
                    ak += ld_dsmem(pk + i * DK + r, g);
                    ag += ld_dsmem(pg + i * DK + r, g);
                }
                const size_t trow = (size_t)(t0 + ts + i) * H + h;
                dq[trow * DK + r] = aq;
                dk[trow * DK + r] = ak;
                dla[trow * DK + r] = ag;
            }
            for (int i = cs * NT + tid; i < nb; i += NCS * NT) {
                float ab = 0.f;
#pragma unroll
                for (int g = 0; g < NCS; ++g) ab += ld_dsmem(pb + i, g);
                dbeta[(size_t)(t0 + ts + i) * H + h] = ab;
            }
        }
    }
    if (dinit) {
#pragma unroll
        for (int m = 0; m < R; ++m) dinit[sbase + el(m)] = dS[m];
    }
    cluster_sync();   // no CTA leaves while another may still read its shared memory
}

// Workspace of the backward: the checkpoints (one d_k x d_v state per chunk of every sequence and
// head) and one chunk's per-token states for every (sequence, head) pair.
inline size_t bwd_workspace_bytes(int64_t N, int64_t H, int64_t total_tokens, int DK, int DV, int C) {
    const size_t kv = (size_t)DK * DV * sizeof(float);
    if (C == 0) return (size_t)H * (size_t)(total_tokens > 0 ? total_tokens : 1) * kv;   // every state
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
    // the checkpoints then the per-pair scratch; with C == 0 only the [H][total tokens] states (the
    // kernel's per-head stride is then total)
    const int64_t nck_head = C == 0 ? total : bwd::ckpts_per_head(total, N, C);
    float *ck = static_cast<float *>(workspace);
    float *scr = C == 0 ? ck : ck + (size_t)H * nck_head * DK * DV;
    const unsigned grid = static_cast<unsigned>(N) * H * SM::NCS;
    if (grid == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(32 * SM::NRG);   // one warp per kRows key rows
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;   // the d_v slices of one (sequence, head)
    attr[0].val.clusterDim.x = SM::NCS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, static_cast<const TIO *>(q), static_cast<const TIO *>(k),
                           static_cast<const TIO *>(v), static_cast<const TIO *>(la), static_cast<const TIO *>(beta),
                           init_state, cu, T, H, C, static_cast<const TDO *>(dout), dfinal, dq, dk, dv, dla, dbeta,
                           dinit, ck, scr, nck_head);
    if (e != cudaSuccess) return e;
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
