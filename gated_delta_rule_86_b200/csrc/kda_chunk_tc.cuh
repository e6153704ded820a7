// kda_chunk_tc.cuh -- chunkwise KDA prefill on the sm_100a tensor cores.
//
// Implements the chunkwise scheme of "Hybrid Linear Attention Architectures:
// Breaking Through the Long-Context Engineering Bottleneck in LLMs" (section
// "Hardware-Aware Chunkwise Parallelism": the inter-chunk state update and the
// intra-chunk output equations; section 3 of "Linear Attention KDA Gating in a
// 3:1 Hybrid Architecture" repeats them with the per-chunk loop).  For a chunk
// of C = 64 tokens with entering state S (d_k x d_v), per key channel c:
//   G_r   = sum_{s<=r} log_alpha_s                  (log-space cumulative decay)
//   A_rs  = beta_r sum_c k_rc k_sc exp(G_rc - G_sc)   for s < r
//   P_rs  =        sum_c q_rc k_sc exp(G_rc - G_sc)   for s <= r
//   T     = (I + A)^{-1}                              (UT transform)
//   W     = T diag(beta) (K * exp(G)),   U = T diag(beta) V      (WY factors)
//   U~    = U - W S
//   O     = (Q * exp(G)) S + P U~
//   S    <- Diag(exp(G_last)) S + (K * exp(G_last - G))^T U~
// which equals the token recurrence exactly in exact arithmetic.
//
// Precision (fp32 accumulation in TMEM, fp32 master state in registers, fp32
// decays and substitution, fp32 or bf16 output):
//   * A and P need the rebased factors below, whose range exceeds fp16: they are
//     bf16 operands, and P (which feeds the output directly) uses a two-term
//     bf16 split of both operands (hi*hi + hi*lo + lo*hi), ~16-bit accuracy.
//   * Every other product (W, U, U~, Q S, P U~, Kd^T U~) has operands bounded by
//     the inputs and runs on fp16 operands (11-bit significand, same tensor
//     rate as bf16).  If any of those values leaves the fp16 range, the chunk's
//     U~ or O turns non-finite; that is detected and the chunk is recomputed on
//     the exact path below.
//
// Exponent range ("log-domain accumulation", section 3 of "Designing and
// Deploying Hybrid MLA and Linear Attention Architectures for LLMs"): the
// products of A and P are formed as (k exp(G - G_ref)) . (k exp(G_ref - G))
// with G_ref the cumulative decay at the chunk's middle token, so each factor
// stays within exp(+-kRangeLimit) whenever the chunk's per-channel decay on
// either side of the middle stays within kRangeLimit.  A chunk whose decays
// exceed that (extremely fast forgetting) is evaluated token by token in fp32
// instead, so every input with finite log_alpha gets a correct result.
//
// Work decomposition: one CTA per (sequence, head, NV-wide slice of d_v).  The
// d_v columns of S evolve independently (column j of U~ depends only on
// column j of S), so slicing d_v multiplies the parallelism of the sequential
// chunk chain; the d_v-independent work (decays, A, P, T, W) is recomputed per
// slice.  Packed variable-length batches are scheduled longest-first.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "kda_recurrent.cuh"
#include "tc_utils.cuh"

namespace kda {

constexpr int kChunk = 64;
constexpr int kDK = 128;
// Largest per-channel cumulative decay (in natural-log units) allowed on either
// side of the chunk's middle token for the tensor-core path.  Factors of the
// rebased products stay within exp(+-40); their sums stay far below the fp32
// and bf16 overflow threshold exp(88.7).
constexpr float kRangeLimit = 40.f;

// ---- shared-memory plan (bytes, all blocks 1024-aligned) ----------------------------------------
template <int NV>
struct ChunkSmem {
    static constexpr int kTile = kChunk * kDK * 2;   // one [64 x 128] 16-bit operand (16 KB)
    // bf16 operands of A_raw and P_raw; dead once those MMAs complete, then
    // reused as fp32 scratch for the UT transform (A and T, 2 x 16 KB).
    static constexpr int kKr = 0;                    // K exp(G - Gref)            A of A_raw
    static constexpr int kQrHi = kKr + kTile;        // Q exp(G - Gref), hi part   A of P_raw
    static constexpr int kQrLo = kQrHi + kTile;      //                 lo part
    static constexpr int kKnHi = kQrLo + kTile;      // K exp(Gref - G), hi part   B of A_raw, P_raw
    static constexpr int kKnLo = kKnHi + kTile;      //                 lo part    B of P_raw
    // fp16 operands
    static constexpr int kKg = kKnLo + kTile;        // K exp(G)                   B of W (MN-major)
    static constexpr int kQg = kKg + kTile;          // Q exp(G)                   A of Q S
    static constexpr int kKd = kQg + kTile;          // K exp(Glast - G)           A of Kd^T U~ (MN-major)
    static constexpr int kT = kKd + kTile;           // T diag(beta) [64 x 64]     A of W, U
    static constexpr int kP = kT + kChunk * kChunk * 2;           // tril(P) [64 x 64]   A of P U~
    static constexpr int kV = kP + kChunk * kChunk * 2;           // V slice [64 x NV]   B of U
    static constexpr int kW = kV + kChunk * NV * 2;               // W [64 x 128]        A of -W S
    static constexpr int kS = kW + kTile;                         // S [128 x NV]        B of W S, Q S
    static constexpr int kUt = kS + kDK * NV * 2;                 // U~ [64 x NV]        B of P U~, Kd^T U~
    static constexpr int kX = kUt + kChunk * NV * 2;              // fp32 [16 x 48] substitution scratch
    static constexpr int kBeta = kX + 16 * 48 * 4;                // fp32 [64]
    static constexpr int kG0 = kBeta + 64 * 4;                    // fp32 [128] decay after token 0
    static constexpr int kGref = kG0 + kDK * 4;                   // fp32 [128] decay after token 31
    static constexpr int kGlast = kGref + kDK * 4;                // fp32 [128] decay after token 63
    static constexpr int kTot = kGlast + kDK * 4;                 // fp32 [8][128] scan totals
    static constexpr int kEnd = kTot + 8 * kDK * 4;
    static constexpr int kBytes = kEnd + 1024;  // + alignment slack
    // exact-path scratch: [128][2 NV] fp32 partial products inside the A/P region
    static_assert(kDK * 2 * NV * 4 <= kKg, "exact-path scratch must fit the A/P operand region");
};

// TMEM columns (fp32 accumulators).  M=64 tiles use lanes 0-15 of each 32-lane
// subpartition (row m -> lane (m % 16) + 32 (m / 16)); M=128 tiles use all lanes.
constexpr uint32_t kTmA = 0, kTmP = 64, kTmSn = 0, kTmW = 128, kTmU = 256, kTmO = 384;
constexpr uint32_t kTmCols = 512;

// Descriptor of k-step `kk` (16 elements along K) of a K-major SW128 operand with `rows` rows.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int rows, int kk) {
    return tc::make_sdesc(base + (kk >> 2) * (rows * 128) + (kk & 3) * 32, 16, 1024, tc::kSwz128);
}
// Descriptor of k-step `kk` of an MN-major operand stored as [K rows x MN columns]:
// SW64 when MN == 32, else 64-column SW128 blocks.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, int krows, int mn, int kk) {
    if (mn == 32) return tc::make_sdesc(base + kk * 1024, krows * 64, 512, tc::kSwz64);
    return tc::make_sdesc(base + kk * 2048, krows * 128, 1024, tc::kSwz128);
}
// Byte offset of 16-byte chunk `j` (8 16-bit columns) of row `r` in a tile with
// `cols` columns stored as above (SW64 for 32 columns, SW128 64-column blocks).
__device__ __forceinline__ uint32_t tile_chunk(int r, int j, int rows, int cols) {
    if (cols == 32) return tc::sw64(r, j);
    return (j >> 3) * (rows * 128) + tc::sw128(r, j & 7);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t pack_h(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ void unpack8(const uint4 &u, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ uint4 pack8_bf16(const float *f) {
    return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
}
__device__ __forceinline__ uint4 pack8_h(const float *f) {
    return make_uint4(pack_h(f[0], f[1]), pack_h(f[2], f[3]), pack_h(f[4], f[5]), pack_h(f[6], f[7]));
}
// bf16 hi part and the bf16 rounding of the remainder (x ~= hi + lo to ~16 bits).
__device__ __forceinline__ void split8_bf16(const float *f, uint4 &hi, uint4 &lo) {
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = f[i] - __bfloat162float(__float2bfloat16_rn(f[i]));
    hi = pack8_bf16(f);
    lo = pack8_bf16(r);
}

template <typename TO> __device__ __forceinline__ void store16(TO *dst, const float *f);
template <> __device__ __forceinline__ void store16<float>(float *dst, const float *f) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        reinterpret_cast<float4 *>(dst)[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
}
template <> __device__ __forceinline__ void store16<__nv_bfloat16>(__nv_bfloat16 *dst, const float *f) {
    reinterpret_cast<uint4 *>(dst)[0] = pack8_bf16(f);
    reinterpret_cast<uint4 *>(dst)[1] = pack8_bf16(f + 8);
}

// Wait for the next completion of the CTA's MMA barrier, then make every
// thread agree on whether the wait succeeded.  Returns false on timeout.
__device__ __forceinline__ bool wait_mma(uint64_t *bar, uint32_t &phase, volatile int *abort_flag) {
    tc::mbar_wait(bar, phase, abort_flag);
    phase ^= 1u;
    tc::tc_fence_after();
    __syncthreads();
    return *abort_flag == 0;
}

template <int NV, typename TO>
__global__ void __launch_bounds__(128, 1)
kda_chunk_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ log_alpha,
                    const __nv_bfloat16 *__restrict__ beta, const float *init_state,
                    const int32_t *__restrict__ cu_seqlens, int num_seqs, int T, int H, int DV,
                    TO *__restrict__ out, float *final_state) {
    using SM = ChunkSmem<NV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    float *sX = reinterpret_cast<float *>(sm + SM::kX);
    float *sBeta = reinterpret_cast<float *>(sm + SM::kBeta);
    float *sG0 = reinterpret_cast<float *>(sm + SM::kG0);
    float *sGref = reinterpret_cast<float *>(sm + SM::kGref);
    float *sGlast = reinterpret_cast<float *>(sm + SM::kGlast);
    float *sTot = reinterpret_cast<float *>(sm + SM::kTot);
    float *sA = reinterpret_cast<float *>(sm + SM::kKr);                   // fp32 [64][64]
    float *sT = reinterpret_cast<float *>(sm + SM::kKr) + kChunk * kChunk;  // fp32 [64][64]

    __shared__ uint64_t bar_mma;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ int s_slot;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nslices = DV / NV;
    const int slice = blockIdx.x % nslices;
    const int pair = blockIdx.x / nslices;
    const int h = pair % H;
    int n = pair / H;
    int64_t t0, t1;
    if (cu_seqlens) {
        if (num_seqs <= kLongestFirstMaxSeqs) n = longest_first_seq(cu_seqlens, num_seqs, n, &s_slot);
        t0 = cu_seqlens[n];
        t1 = cu_seqlens[n + 1];
    } else {
        t0 = (int64_t)n * T;
        t1 = t0 + T;
    }
    const int64_t len = t1 - t0;
    const int nchunks = static_cast<int>((len + kChunk - 1) / kChunk);
    const int vcol0 = slice * NV;  // first value column of this slice

    if (tid == 0) {
        tc::mbar_init(&bar_mma, 1);
        tc::fence_mbar_init();
        abort_flag = 0;
    }
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base_sh, kTmCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    const uint32_t tl = tc::tmem_lane_base(warp);
    uint32_t phase = 0;

    // ---- fp32 master state: thread i owns key row i, NV value columns -----------------------------
    float S[NV];
    const size_t state_base = ((size_t)n * H + h) * kDK * DV;
#pragma unroll
    for (int j = 0; j < NV; ++j) S[j] = init_state ? init_state[state_base + (size_t)tid * DV + vcol0 + j] : 0.f;

    // fp16 copy of S as the MN-major B operand [128 K-rows x NV]
    auto write_state_operand = [&]() {
#pragma unroll
        for (int j = 0; j < NV / 8; ++j)
            *reinterpret_cast<uint4 *>(sm + SM::kS + tile_chunk(tid, j, kDK, NV)) = pack8_h(&S[8 * j]);
    };
    write_state_operand();

    // Exact evaluation of one chunk, token by token in fp32 (the recurrence
    // itself), starting from the state in registers.  Used when the chunk's
    // decays exceed the rebasing range or an fp16 operand overflowed.
    auto exact_chunk = [&](int64_t tok0, int L) {
        float *red = reinterpret_cast<float *>(sm + SM::kKr);  // [128][2 NV]
        float *col = reinterpret_cast<float *>(sm + SM::kKg);  // [2 NV]
        for (int r = 0; r < L; ++r) {
            const int64_t row = (tok0 + r) * H + h;
            const float a = expf(__bfloat162float(log_alpha[row * kDK + tid]));
            const float kk = __bfloat162float(k[row * kDK + tid]);
            const float qq = __bfloat162float(q[row * kDK + tid]);
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                S[j] *= a;
                red[tid * (2 * NV) + j] = S[j] * kk;
                red[tid * (2 * NV) + NV + j] = S[j] * qq;
            }
            float kq = kk * qq;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
            if (lane == 0) sX[warp] = kq;
            __syncthreads();
            if (tid < 2 * NV) {
                float acc = 0.f;
                for (int i = 0; i < kDK; ++i) acc += red[i * (2 * NV) + tid];
                col[tid] = acc;
            }
            __syncthreads();
            const float kqs = sX[0] + sX[1] + sX[2] + sX[3];
            const float b = __bfloat162float(beta[row]);
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const float u = b * (__bfloat162float(v[row * DV + vcol0 + j]) - col[j]);
                if (tid == j) out[row * DV + vcol0 + j] = from_f32<TO>(fmaf(u, kqs, col[NV + j]));
                S[j] = fmaf(kk, u, S[j]);
            }
            __syncthreads();
        }
        write_state_operand();
        __syncthreads();
    };

    for (int c = 0; c < nchunks; ++c) {
        const int64_t tok0 = t0 + (int64_t)c * kChunk;  // first token of the chunk
        const int L = static_cast<int>((t1 - tok0) < kChunk ? (t1 - tok0) : kChunk);

        // ================= phase E: decays, range check, rebased operands =================
        const int cg = tid & 15, tg = tid >> 4;  // 8 channels [8cg, 8cg+8), 8 tokens [8tg, 8tg+8)
        float G[8][8];                            // cumulative decay, this thread's 8 x 8 block
        {
            float run[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) run[i] = 0.f;
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                const int r = tg * 8 + rr;
                float g8[8];
                if (r < L) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(log_alpha + ((tok0 + r) * H + h) * kDK + cg * 8);
                    unpack8(u, g8);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) g8[i] = 0.f;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    run[i] += g8[i];
                    G[rr][i] = run[i];
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) sTot[tg * kDK + cg * 8 + i] = run[i];
            __syncthreads();
            float off[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) off[i] = 0.f;
            for (int p = 0; p < tg; ++p)
#pragma unroll
                for (int i = 0; i < 8; ++i) off[i] += sTot[p * kDK + cg * 8 + i];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr)
#pragma unroll
                for (int i = 0; i < 8; ++i) G[rr][i] += off[i];
            // decays after tokens 0, 31 and 63 (padding rows carry log_alpha = 0)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (tg == 0) sG0[cg * 8 + i] = G[0][i];
                if (tg == 3) sGref[cg * 8 + i] = G[7][i];
                if (tg == 7) sGlast[cg * 8 + i] = G[7][i];
            }
        }
        if (tid < 64) sBeta[tid] = (tid < L) ? __bfloat162float(beta[(tok0 + tid) * H + h]) : 0.f;
        __syncthreads();
        {
            const float g0 = sG0[tid], gr = sGref[tid], gl = sGlast[tid];
            const bool bad = !((g0 - gr <= kRangeLimit) && (gr - gl <= kRangeLimit));
            if (__syncthreads_or(bad)) {
                exact_chunk(tok0, L);
                continue;
            }
        }
        {
            float gref[8], erefabs[8], elast[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                gref[i] = sGref[cg * 8 + i];
                erefabs[i] = expf(gref[i]);                       // exp(Gref)
                elast[i] = expf(sGlast[cg * 8 + i] - gref[i]);   // exp(Glast - Gref)
            }
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                const int r = tg * 8 + rr;
                float kf[8], qf[8];
                if (r < L) {
                    const int64_t row = (tok0 + r) * H + h;
                    unpack8(*reinterpret_cast<const uint4 *>(k + row * kDK + cg * 8), kf);
                    unpack8(*reinterpret_cast<const uint4 *>(q + row * kDK + cg * 8), qf);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) kf[i] = qf[i] = 0.f;
                }
                float kr[8], qr[8], kn[8], kg[8], qg[8], kd[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float dg = G[rr][i] - gref[i];
                    const float e1 = fast_exp(dg), e2 = fast_exp(-dg);
                    kr[i] = kf[i] * e1;
                    qr[i] = qf[i] * e1;
                    kn[i] = kf[i] * e2;
                    kg[i] = kr[i] * erefabs[i];
                    qg[i] = qr[i] * erefabs[i];
                    kd[i] = kn[i] * elast[i];
                }
                const uint32_t off = tile_chunk(r, cg, kChunk, kDK);
                uint4 hi, lo;
                *reinterpret_cast<uint4 *>(sm + SM::kKr + off) = pack8_bf16(kr);
                split8_bf16(qr, hi, lo);
                *reinterpret_cast<uint4 *>(sm + SM::kQrHi + off) = hi;
                *reinterpret_cast<uint4 *>(sm + SM::kQrLo + off) = lo;
                split8_bf16(kn, hi, lo);
                *reinterpret_cast<uint4 *>(sm + SM::kKnHi + off) = hi;
                *reinterpret_cast<uint4 *>(sm + SM::kKnLo + off) = lo;
                *reinterpret_cast<uint4 *>(sm + SM::kKg + off) = pack8_h(kg);
                *reinterpret_cast<uint4 *>(sm + SM::kQg + off) = pack8_h(qg);
                *reinterpret_cast<uint4 *>(sm + SM::kKd + off) = pack8_h(kd);
            }
            // V slice [64 x NV] (fp16) as the MN-major B operand of U
            for (int idx = tid; idx < kChunk * (NV / 8); idx += 128) {
                const int r = idx / (NV / 8), j = idx % (NV / 8);
                float f[8];
                if (r < L) {
                    unpack8(*reinterpret_cast<const uint4 *>(v + ((tok0 + r) * H + h) * DV + vcol0 + j * 8), f);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) f[i] = 0.f;
                }
                *reinterpret_cast<uint4 *>(sm + SM::kV + tile_chunk(r, j, kChunk, NV)) = pack8_h(f);
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // ================= M1: A_raw = Kr Kn^T,  P_raw = Qr Kn^T (split) =================
        if (tid == 0) {
            tc::tc_fence_after();
            constexpr uint32_t id = tc::make_idesc(64, 64, tc::kBF16, false, false);
#pragma unroll
            for (int kk = 0; kk < kDK / 16; ++kk) {
                const uint64_t bhi = desc_kmajor(sbase + SM::kKnHi, kChunk, kk);
                const uint64_t blo = desc_kmajor(sbase + SM::kKnLo, kChunk, kk);
                const uint64_t qhi = desc_kmajor(sbase + SM::kQrHi, kChunk, kk);
                tc::mma_f16(tmem + kTmA, desc_kmajor(sbase + SM::kKr, kChunk, kk), bhi, id, kk > 0);
                tc::mma_f16(tmem + kTmP, qhi, bhi, id, kk > 0);
                tc::mma_f16(tmem + kTmP, qhi, blo, id, true);
                tc::mma_f16(tmem + kTmP, desc_kmajor(sbase + SM::kQrLo, kChunk, kk), bhi, id, true);
            }
            tc::mma_commit(&bar_mma);
        }
        if (!wait_mma(&bar_mma, phase, &abort_flag)) break;

        // ================= phase S: masks, UT transform =================
        {
            const bool owner = lane < 16;
            const int r = warp * 16 + lane;
            float a16[16], p16[16];
#pragma unroll
            for (int c16 = 0; c16 < 4; ++c16) {
                tc::tmem_ld16(tmem + tl + kTmA + c16 * 16, a16);
                tc::tmem_ld16(tmem + tl + kTmP + c16 * 16, p16);
                tc::tmem_ld_wait();
                if (owner) {
                    const float br = sBeta[r];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int s = c16 * 16 + i;
                        sA[r * kChunk + s] = (s < r) ? br * a16[i] : 0.f;
                        p16[i] = (s <= r) ? p16[i] : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(sm + SM::kP + tile_chunk(r, 2 * c16, kChunk, kChunk)) = pack8_h(p16);
                    *reinterpret_cast<uint4 *>(sm + SM::kP + tile_chunk(r, 2 * c16 + 1, kChunk, kChunk)) =
                        pack8_h(p16 + 8);
                }
            }
            for (int i = tid; i < kChunk * kChunk; i += 128) sT[i] = 0.f;
        }
        tc::tc_fence_before();
        __syncthreads();
        // diagonal 16x16 blocks: thread (b, cc) computes column cc of (I + A_bb)^{-1}
        if (tid < 64) {
            const int b = tid >> 4, cc = tid & 15;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int s = 0; s < 15; ++s)
                    if (s < r && s >= cc) acc = fmaf(sA[(16 * b + r) * kChunk + 16 * b + s], x[s], acc);
                x[r] = (r == cc) ? 1.f : ((r > cc) ? -acc : 0.f);
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) sT[(16 * b + r) * kChunk + 16 * b + cc] = x[r];
        }
        __syncthreads();
        // off-diagonal row blocks: T[i, 0:16i] = -D_i (A[i, 0:16i] T[0:16i, 0:16i])
        for (int ib = 1; ib < 4; ++ib) {
            const int w = 16 * ib;
            for (int e = tid; e < 16 * w; e += 128) {
                const int r = e / w, cc = e % w;
                float acc = 0.f;
                for (int m = cc; m < w; ++m) acc = fmaf(sA[(w + r) * kChunk + m], sT[m * kChunk + cc], acc);
                sX[r * 48 + cc] = acc;
            }
            __syncthreads();
            for (int e = tid; e < 16 * w; e += 128) {
                const int r = e / w, cc = e % w;
                float acc = 0.f;
                for (int m = 0; m <= r; ++m) acc = fmaf(sT[(w + r) * kChunk + w + m], sX[m * 48 + cc], acc);
                sT[(w + r) * kChunk + cc] = -acc;
            }
            __syncthreads();
        }
        // T diag(beta) -> fp16 A operand [64 x 64]
        {
            const int r = tid >> 1, half = tid & 1;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int s = half * 32 + j * 8 + i;
                    f[i] = sT[r * kChunk + s] * sBeta[s];
                }
                *reinterpret_cast<uint4 *>(sm + SM::kT + tile_chunk(r, half * 4 + j, kChunk, kChunk)) = pack8_h(f);
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // ================= M2: W = (T b) Kg,  U = (T b) V =================
        if (tid == 0) {
            tc::tc_fence_after();
            constexpr uint32_t idW = tc::make_idesc(64, kDK, tc::kF16, false, true);
            constexpr uint32_t idU = tc::make_idesc(64, NV, tc::kF16, false, true);
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk) {
                const uint64_t adesc = desc_kmajor(sbase + SM::kT, kChunk, kk);
                tc::mma_f16(tmem + kTmW, adesc, desc_mnmajor(sbase + SM::kKg, kChunk, kDK, kk), idW, kk > 0);
                tc::mma_f16(tmem + kTmU, adesc, desc_mnmajor(sbase + SM::kV, kChunk, NV, kk), idU, kk > 0);
            }
            tc::mma_commit(&bar_mma);
        }
        if (!wait_mma(&bar_mma, phase, &abort_flag)) break;

        // W -> fp16 A operand [64 x 128]
        {
            const bool owner = lane < 16;
            const int r = warp * 16 + lane;
#pragma unroll
            for (int c16 = 0; c16 < kDK / 16; ++c16) {
                float w16[16];
                tc::tmem_ld16(tmem + tl + kTmW + c16 * 16, w16);
                tc::tmem_ld_wait();
                if (owner) {
                    *reinterpret_cast<uint4 *>(sm + SM::kW + tile_chunk(r, 2 * c16, kChunk, kDK)) = pack8_h(w16);
                    *reinterpret_cast<uint4 *>(sm + SM::kW + tile_chunk(r, 2 * c16 + 1, kChunk, kDK)) =
                        pack8_h(w16 + 8);
                }
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();

        // ================= M3: U~ = U - W S (into U),  O = Qg S =================
        if (tid == 0) {
            tc::tc_fence_after();
            constexpr uint32_t idNeg = tc::make_idesc(64, NV, tc::kF16, false, true, true);
            constexpr uint32_t idO = tc::make_idesc(64, NV, tc::kF16, false, true);
#pragma unroll
            for (int kk = 0; kk < kDK / 16; ++kk) {
                const uint64_t bdesc = desc_mnmajor(sbase + SM::kS, kDK, NV, kk);
                tc::mma_f16(tmem + kTmU, desc_kmajor(sbase + SM::kW, kChunk, kk), bdesc, idNeg, true);
                tc::mma_f16(tmem + kTmO, desc_kmajor(sbase + SM::kQg, kChunk, kk), bdesc, idO, kk > 0);
            }
            tc::mma_commit(&bar_mma);
        }
        if (!wait_mma(&bar_mma, phase, &abort_flag)) break;

        // U~ -> fp16 MN-major B operand [64 x NV]; a value outside the fp16
        // range sends the chunk to the exact path
        {
            const bool owner = lane < 16;
            const int r = warp * 16 + lane;
            bool bad = false;
#pragma unroll
            for (int c16 = 0; c16 < NV / 16; ++c16) {
                float u16[16];
                tc::tmem_ld16(tmem + tl + kTmU + c16 * 16, u16);
                tc::tmem_ld_wait();
                if (owner) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) bad |= !(fabsf(u16[i]) <= 65000.f);
                    *reinterpret_cast<uint4 *>(sm + SM::kUt + tile_chunk(r, 2 * c16, kChunk, NV)) = pack8_h(u16);
                    *reinterpret_cast<uint4 *>(sm + SM::kUt + tile_chunk(r, 2 * c16 + 1, kChunk, NV)) =
                        pack8_h(u16 + 8);
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            if (__syncthreads_or(bad)) {
                exact_chunk(tok0, L);
                continue;
            }
        }

        // ================= M4: O += P U~,  Sn = Kd^T U~ =================
        if (tid == 0) {
            tc::tc_fence_after();
            constexpr uint32_t idO = tc::make_idesc(64, NV, tc::kF16, false, true);
            constexpr uint32_t idS = tc::make_idesc(128, NV, tc::kF16, true, true);
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk) {
                const uint64_t bdesc = desc_mnmajor(sbase + SM::kUt, kChunk, NV, kk);
                tc::mma_f16(tmem + kTmO, desc_kmajor(sbase + SM::kP, kChunk, kk), bdesc, idO, true);
                tc::mma_f16(tmem + kTmSn, desc_mnmajor(sbase + SM::kKd, kChunk, kDK, kk), bdesc, idS, kk > 0);
            }
            tc::mma_commit(&bar_mma);
        }
        if (!wait_mma(&bar_mma, phase, &abort_flag)) break;

        // ================= epilogue: output rows, state update =================
        {
            const bool owner = lane < 16;
            const int r = warp * 16 + lane;
            float o[NV];
            bool bad = false;
#pragma unroll
            for (int c16 = 0; c16 < NV / 16; ++c16) {
                float o16[16];
                tc::tmem_ld16(tmem + tl + kTmO + c16 * 16, o16);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) o[c16 * 16 + i] = o16[i];
            }
            if (owner)
#pragma unroll
                for (int i = 0; i < NV; ++i) bad |= !(fabsf(o[i]) <= 3.0e38f);
            tc::tc_fence_before();
            if (__syncthreads_or(bad)) {
                exact_chunk(tok0, L);
                continue;
            }
            if (owner && r < L) {
                TO *dst = out + ((tok0 + r) * H + h) * DV + vcol0;
#pragma unroll
                for (int c16 = 0; c16 < NV / 16; ++c16) store16<TO>(dst + c16 * 16, &o[c16 * 16]);
            }
            const float gam = expf(sGlast[tid]);
#pragma unroll
            for (int c16 = 0; c16 < NV / 16; ++c16) {
                float s16[16];
                tc::tmem_ld16(tmem + tl + kTmSn + c16 * 16, s16);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) S[c16 * 16 + i] = fmaf(gam, S[c16 * 16 + i], s16[i]);
            }
            write_state_operand();
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncthreads();
    }

    if (final_state && abort_flag == 0) {
#pragma unroll
        for (int j = 0; j < NV; ++j) final_state[state_base + (size_t)tid * DV + vcol0 + j] = S[j];
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmCols);
}

template <int NV, typename TO>
cudaError_t launch_chunk_tc_nv(const void *q, const void *k, const void *v, const void *la, const void *beta,
                               const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H, int DV,
                               void *out, float *final_state, cudaStream_t stream) {
    auto kern = kda_chunk_tc_kernel<NV, TO>;
    const int smem = ChunkSmem<NV>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int N = cu ? num_seqs : B;
    const unsigned grid = static_cast<unsigned>(N) * H * (DV / NV);
    kern<<<grid, 128, smem, stream>>>(static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
                                      static_cast<const __nv_bfloat16 *>(v), static_cast<const __nv_bfloat16 *>(la),
                                      static_cast<const __nv_bfloat16 *>(beta), init_state, cu, num_seqs, T, H, DV,
                                      static_cast<TO *>(out), final_state);
    return cudaGetLastError();
}

// Slice width: narrow slices when there are few (sequence, head) pairs, so the
// grid still covers the SMs.
template <typename TO>
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const void *la, const void *beta,
                            const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H, int DV,
                            void *out, float *final_state, cudaStream_t stream) {
    const int64_t pairs = (int64_t)(cu ? num_seqs : B) * H;
    if (pairs * (DV / 64) < 148)
        return launch_chunk_tc_nv<32, TO>(q, k, v, la, beta, init_state, cu, num_seqs, B, T, H, DV, out, final_state,
                                          stream);
    return launch_chunk_tc_nv<64, TO>(q, k, v, la, beta, init_state, cu, num_seqs, B, T, H, DV, out, final_state,
                                      stream);
}

}  // namespace kda
