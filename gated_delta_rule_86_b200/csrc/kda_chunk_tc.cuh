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
// Pipeline.  Everything up to W and U depends only on the chunk's own inputs;
// only the last three lines touch S.  One cluster of CL = d_v / 32 CTAs handles
// one (sequence, head); CTA r owns value columns [32 r, 32 r + 32) and runs
// three roles:
//   * prep (warps 4-11): for every CL-th chunk (c = r mod CL): decays, rebased
//     operands, A/P, UT transform and W.  The finished operands of the chunk
//     (Kd, P, Qg, W, T diag(beta), gamma and a flag) form one contiguous image,
//     which is bulk-stored to a per-producer region of a global workspace and
//     announced to every CTA of the cluster through remote mbarrier arrives;
//   * chain (warps 0-3): for every chunk, bulk-loads the image (in two parts,
//     so the next chunk's loads overlap this chunk's MMAs), computes U on its
//     own value slice, then the state-dependent MMAs, output rows and the fp32
//     state update, and tells the producer when the region may be reused.
// The prep of a chunk is thus computed once per head instead of once per
// slice, and each CTA spends only 1/CL of its time on it.

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
// Work decomposition: the d_v columns of S evolve independently (column j of U~
// depends only on column j of S), so slicing d_v across the CTAs of a cluster
// multiplies the parallelism of the sequential chunk chain.  Packed
// variable-length batches are scheduled longest-first.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "kda_recurrent.cuh"
#include "tc_utils.cuh"

namespace kda {

constexpr int kChunk = 64;
constexpr int kDK = 128;
constexpr int kNV = 32;  // value columns per CTA
// Largest per-channel cumulative decay (in natural-log units) allowed on either
// side of the chunk's middle token for the tensor-core path.  Factors of the
// rebased products stay within exp(+-40); their sums stay far below the fp32
// and bf16 overflow threshold exp(88.7).
constexpr float kRangeLimit = 40.f;

constexpr int kChainThreads = 128;  // warps 0-3
constexpr int kPrepThreads = 256;   // warps 4-11
constexpr int kThreads = kChainThreads + kPrepThreads;
constexpr uint32_t kBarPrep = 1, kBarChain = 2;  // named barrier ids

// ---- chunk image: the prep results of one chunk, in their MMA layouts (fp16) -----------------
// part 2 (consumed by the second chain MMA group) first, part 1 after it.
struct ChunkImage {
    static constexpr int kTile = kChunk * kDK * 2;      // [64 x 128] 16-bit tile
    static constexpr int kKd = 0;                       // K exp(Glast - G)   A of Kd^T U~ (MN-major)
    static constexpr int kP = kKd + kTile;              // tril(P) [64 x 64]  A of P U~
    static constexpr int kPart1 = kP + kChunk * kChunk * 2;
    static constexpr int kQg = kPart1;                  // Q exp(G)           A of Q S
    static constexpr int kW = kQg + kTile;              // W [64 x 128]       A of -W S
    static constexpr int kTb = kW + kTile;              // T diag(beta)       A of U
    static constexpr int kGamma = kTb + kChunk * kChunk * 2;   // fp32 [128] exp(Glast)
    static constexpr int kFlag = kGamma + kDK * 4;             // int: 1 = evaluate exactly
    static constexpr int kBytes = kFlag + 16;
    static constexpr int kPart2Bytes = kPart1;
    static constexpr int kPart1Bytes = kBytes - kPart1;
    static constexpr int kStride = (kBytes + 1023) / 1024 * 1024;  // workspace region stride
};

// ---- shared-memory plan (byte offsets; operand tiles 1024-aligned) -------------------------------
struct ChunkSmem {
    using I = ChunkImage;
    static constexpr int kTile = I::kTile;
    // prep region: the image of the chunk being prepared, and its scratch
    static constexpr int kImg = 0;
    // bf16 operands of A_raw and P_raw (dead once those MMAs complete); they
    // overlap the image's W/Tb/gamma/flag, which are written later
    static constexpr int kKr = I::kW;                 // K exp(G - Gref)            A of A_raw
    static constexpr int kQrHi = kKr + kTile;         // Q exp(G - Gref), hi        A of P_raw
    static constexpr int kQrLo = kQrHi + kTile;       //                  lo
    static constexpr int kKnHi = kQrLo + kTile;       // K exp(Gref - G), hi        B of A_raw, P_raw
    static constexpr int kKnLo = kKnHi + kTile;       //                  lo
    static constexpr int kApEnd = kKnLo + kTile;
    // fp32 scratch of the UT transform, inside the dead A/P operands and past the image
    static constexpr int kLd = 68;                    // fp32 row stride of A and T (bank spread, 16-B rows)
    static constexpr int kA32 = (I::kBytes + 1023) / 1024 * 1024 + 7168;
    static constexpr int kT32 = kA32 + kChunk * kLd * 4;
    static constexpr int kX32 = kT32 + kChunk * kLd * 4;      // fp32 [3][16][16] block products
    static constexpr int kTot = kA32;                          // fp32 [8][128] scan totals (decay phase only)
    static constexpr int kKg = kApEnd;                // K exp(G) [64 x 128]        B of W (MN-major)
    static constexpr int kPrepEnd = kKg + kTile;
    // chain region
    static constexpr int kSlot = kPrepEnd;            // the chain's copy of the current chunk image
    static constexpr int kV = kSlot + I::kStride;     // V slice [64 x 32] fp16   B of U
    static constexpr int kS = kV + kChunk * kNV * 2;  // S [128 x 32] fp16        B of W S, Q S
    static constexpr int kUt = kS + kDK * kNV * 2;    // U~ [64 x 32] fp16        B of P U~, Kd^T U~
    // small fp32 arrays
    static constexpr int kBeta = kUt + kChunk * kNV * 2;      // [64]  prep
    static constexpr int kG0 = kBeta + kChunk * 4;            // [128] decay after token 0
    static constexpr int kGref = kG0 + kDK * 4;               // [128] decay after token 31
    static constexpr int kGlast = kGref + kDK * 4;            // [128] decay after token 63
    static constexpr int kRed = kGlast + kDK * 4;             // chain exact path: 292 floats
    static constexpr int kEnd = kRed + 300 * 4;
    static constexpr int kBytes = kEnd + 1024;                // + alignment slack
    static_assert(kX32 + 3 * 256 * 4 <= kApEnd, "UT scratch must fit the dead A/P operands");
    static_assert(kTot + 8 * kDK * 4 <= kApEnd, "scan totals must fit the dead A/P operands");
    static_assert(kBytes <= 232448, "shared memory plan exceeds 227 KB");
};

// TMEM columns (fp32 accumulators).  M=64 tiles use lanes 0-15 of each 32-lane
// subpartition (row m -> lane (m % 16) + 32 (m / 16)); M=128 tiles use all lanes.
constexpr uint32_t kTmA = 0, kTmP = 64, kTmW = 128, kTmU = 256, kTmO = 288, kTmSn = 320;
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
// Two-term bf16 split x ~= hi + lo: hi is x truncated to bf16 (exact in fp32),
// lo the bf16 rounding of the exact remainder; |x - hi - lo| <= 2^-15 |x|.
__device__ __forceinline__ void split8_bf16(const float *f, uint4 &hi, uint4 &lo) {
    float r[8];
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = f[i] - __uint_as_float(__float_as_uint(f[i]) & 0xffff0000u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __byte_perm(__float_as_uint(f[2 * i]), __float_as_uint(f[2 * i + 1]), 0x7632);
    hi = make_uint4(h[0], h[1], h[2], h[3]);
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

// Sum 32 per-lane values across the warp so that lane l ends with the warp-wide
// sum of value l (recursive halving: 31 shuffles for 32 values).
__device__ __forceinline__ void warp_transpose_sum32(float (&v)[32], int lane) {
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
}

// One thread of a role waits on an mbarrier phase (bounded), then the role's
// named barrier spreads the outcome.  Returns false on timeout or abort.
__device__ __forceinline__ bool role_wait(uint64_t *bar, uint32_t parity, bool leader, uint32_t bar_id,
                                          uint32_t nthreads, volatile int *abort_flag) {
    bool ok = true;
    if (leader) ok = tc::mbar_wait(bar, parity, abort_flag);
    const bool failed = tc::named_sync_or(bar_id, nthreads, !ok);
    tc::tc_fence_after();
    return !failed;
}

template <int CL, typename TO>
__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ log_alpha,
                    const __nv_bfloat16 *__restrict__ beta, const float *init_state,
                    const int32_t *__restrict__ cu_seqlens, int num_seqs, int T, int H, int DV,
                    TO *__restrict__ out, float *final_state, uint8_t *__restrict__ workspace) {
    using SM = ChunkSmem;
    using I = ChunkImage;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    float *sBeta = reinterpret_cast<float *>(sm + SM::kBeta);
    float *sG0 = reinterpret_cast<float *>(sm + SM::kG0);
    float *sGref = reinterpret_cast<float *>(sm + SM::kGref);
    float *sGlast = reinterpret_cast<float *>(sm + SM::kGlast);
    float *sTot = reinterpret_cast<float *>(sm + SM::kTot);
    float *sRed = reinterpret_cast<float *>(sm + SM::kRed);

    // chain: bar_m3, bar_m4 (MMA completion), full1/full2 (image part loads), pub[p] (chunk of
    // producer p stored); prep: bar_m1, bar_m2 (MMA completion), consumed (all CL chains loaded
    // this producer's last chunk)
    __shared__ uint64_t bar_m1, bar_m2, bar_m3, bar_m4, full1, full2, consumed, pub[CL];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ int s_slot;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = static_cast<int>(tc::cluster_ctarank());   // == value slice
    const int pair = blockIdx.x / CL;
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
    const int nchunks = static_cast<int>((t1 - t0 + kChunk - 1) / kChunk);
    const int vcol0 = rank * kNV;
    uint8_t *ws_cluster = workspace + (size_t)pair * CL * I::kStride;  // CL producer regions

    if (tid == 0) {
        tc::mbar_init(&bar_m1, 1);
        tc::mbar_init(&bar_m2, 1);
        tc::mbar_init(&bar_m3, 1);
        tc::mbar_init(&bar_m4, 1);
        tc::mbar_init(&full1, 1);
        tc::mbar_init(&full2, 1);
        tc::mbar_init(&consumed, CL);
        for (int p = 0; p < CL; ++p) tc::mbar_init(&pub[p], 1);
        tc::fence_mbar_init();
        abort_flag = 0;
    }
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base_sh, kTmCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync();  // every CTA's barriers are initialised before any remote arrive
    tc::tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    const uint32_t tl = tc::tmem_lane_base(warp);

    if (warp < 4) {
        // ===================================== chain role =====================================
        const bool leader = tid == 0;
        uint8_t *slot = sm + SM::kSlot;
        const float *sGam = reinterpret_cast<const float *>(slot + I::kGamma);
        const volatile int *sFlag = reinterpret_cast<const volatile int *>(slot + I::kFlag);
        float S[kNV];  // fp32 master state: key row tid, this slice's value columns
        const size_t state_base = ((size_t)n * H + h) * kDK * DV + (size_t)tid * DV + vcol0;
#pragma unroll
        for (int j = 0; j < kNV; ++j) S[j] = init_state ? init_state[state_base + j] : 0.f;
        auto write_state_operand = [&]() {
#pragma unroll
            for (int j = 0; j < kNV / 8; ++j)
                *reinterpret_cast<uint4 *>(sm + SM::kS + tile_chunk(tid, j, kDK, kNV)) = pack8_h(&S[8 * j]);
            tc::fence_async_smem();
        };
        write_state_operand();

        // V slice of a chunk: 64 rows x 4 chunks of 8 values, two per thread, prefetched a chunk ahead
        uint4 rv[2];
        auto load_v = [&](int c) {
            const int64_t tok0 = t0 + (int64_t)c * kChunk;
            const int L = static_cast<int>((t1 - tok0) < kChunk ? (t1 - tok0) : kChunk);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int idx = tid + e * kChainThreads, r = idx >> 2, j = idx & 3;
                rv[e] = (r < L) ? *reinterpret_cast<const uint4 *>(v + ((tok0 + r) * H + h) * DV + vcol0 + j * 8)
                                : make_uint4(0, 0, 0, 0);
            }
        };

        // token-by-token fp32 evaluation of one chunk from the state in registers
        auto exact_chunk = [&](int64_t tok0, int L) {
            for (int r = 0; r < L; ++r) {
                const int64_t row = (tok0 + r) * H + h;
                const float a = expf(__bfloat162float(log_alpha[row * kDK + tid]));
                const float kk = __bfloat162float(k[row * kDK + tid]);
                const float qq = __bfloat162float(q[row * kDK + tid]);
                float va[32], vb[32];
#pragma unroll
                for (int j = 0; j < kNV; ++j) {
                    S[j] *= a;
                    va[j] = S[j] * kk;
                    vb[j] = S[j] * qq;
                }
                warp_transpose_sum32(va, lane);
                warp_transpose_sum32(vb, lane);
                float kq = kk * qq;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
                sRed[warp * 64 + lane] = va[0];
                sRed[warp * 64 + 32 + lane] = vb[0];
                if (lane == 0) sRed[256 + warp] = kq;
                tc::named_sync(kBarChain, kChainThreads);
                if (warp == 0) {
                    float aa = 0.f, bb = 0.f, kqs = 0.f;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        aa += sRed[w * 64 + lane];
                        bb += sRed[w * 64 + 32 + lane];
                        kqs += sRed[256 + w];
                    }
                    const float u = __bfloat162float(beta[row]) *
                                    (__bfloat162float(v[row * DV + vcol0 + lane]) - aa);
                    sRed[260 + lane] = u;
                    out[row * DV + vcol0 + lane] = from_f32<TO>(fmaf(u, kqs, bb));
                }
                tc::named_sync(kBarChain, kChainThreads);
#pragma unroll
                for (int j = 0; j < kNV; ++j) S[j] = fmaf(kk, sRed[260 + j], S[j]);
                tc::named_sync(kBarChain, kChainThreads);
            }
            write_state_operand();
        };

        // image loads (leader only): part 1 = Qg, W, Tb, gamma, flag; part 2 = Kd, P
        auto region = [&](int c) -> const uint8_t * { return ws_cluster + (size_t)(c % CL) * I::kStride; };
        auto issue_part1 = [&](int c) {
            tc::mbar_arrive_expect_tx(&full1, I::kPart1Bytes);
            tc::bulk_load(slot + I::kPart1, region(c) + I::kPart1, I::kPart1Bytes, &full1);
        };
        auto issue_part2 = [&](int c) {
            tc::mbar_arrive_expect_tx(&full2, I::kPart2Bytes);
            tc::bulk_load(slot, region(c), I::kPart2Bytes, &full2);
        };
        bool pre1 = false, pre2 = false;  // parts of the next chunk already issued (leader's view)

        uint32_t ph_m3 = 0, ph_m4 = 0;
        if (nchunks > 0) load_v(0);
        tc::named_sync(kBarChain, kChainThreads);
        for (int c = 0; c < nchunks; ++c) {
            const int64_t tok0 = t0 + (int64_t)c * kChunk;
            const int L = static_cast<int>((t1 - tok0) < kChunk ? (t1 - tok0) : kChunk);
            const int prod = c % CL;
            // ---- make sure this chunk's image loads are in flight ----
            if (leader && !(pre1 && pre2)) {
                bool ok = true;
                if (!pre1) {
                    ok = tc::mbar_wait_cluster(&pub[prod], (c / CL) & 1, &abort_flag);
                    tc::fence_async_global();
                    if (ok) issue_part1(c);
                }
                if (ok && !pre2) issue_part2(c);
            }
            pre1 = pre2 = false;
            // V slice of this chunk (the previous chunk's U MMA has completed)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int idx = tid + e * kChainThreads;
                float f[8];
                unpack8(rv[e], f);
                *reinterpret_cast<uint4 *>(sm + SM::kV + tile_chunk(idx >> 2, idx & 3, kChunk, kNV)) = pack8_h(f);
            }
            tc::fence_async_smem();
            if (c + 1 < nchunks) load_v(c + 1);
            if (!role_wait(&full1, c & 1, leader, kBarChain, kChainThreads, &abort_flag)) break;
            const bool exact = *sFlag != 0;
            const float gam = sGam[tid];
            bool bad = exact;
            bool part2_done = false;
            if (!exact) {
                // ---- M3: U = Tb V;  U~ = U - W S;  O = Qg S ----
                if (leader) {
                    constexpr uint32_t idU = tc::make_idesc(64, kNV, tc::kF16, false, true);
                    constexpr uint32_t idNeg = tc::make_idesc(64, kNV, tc::kF16, false, true, true);
                    constexpr uint32_t idO = tc::make_idesc(64, kNV, tc::kF16, false, true);
#pragma unroll
                    for (int kk = 0; kk < kChunk / 16; ++kk)
                        tc::mma_f16(tmem + kTmU, desc_kmajor(sbase + SM::kSlot + I::kTb, kChunk, kk),
                                    desc_mnmajor(sbase + SM::kV, kChunk, kNV, kk), idU, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < kDK / 16; ++kk) {
                        const uint64_t bdesc = desc_mnmajor(sbase + SM::kS, kDK, kNV, kk);
                        tc::mma_f16(tmem + kTmU, desc_kmajor(sbase + SM::kSlot + I::kW, kChunk, kk), bdesc, idNeg,
                                    true);
                        tc::mma_f16(tmem + kTmO, desc_kmajor(sbase + SM::kSlot + I::kQg, kChunk, kk), bdesc, idO,
                                    kk > 0);
                    }
                    tc::mma_commit(&bar_m3);
                }
                if (!role_wait(&bar_m3, ph_m3, leader, kBarChain, kChainThreads, &abort_flag)) break;
                ph_m3 ^= 1u;
                // part 1 of the image has been read: start loading the next chunk's part 1
                if (leader && c + 1 < nchunks &&
                    tc::mbar_test_wait_cluster(&pub[(c + 1) % CL], ((c + 1) / CL) & 1)) {
                    tc::fence_async_global();
                    issue_part1(c + 1);
                    pre1 = true;
                }
                // U~ -> fp16 B operand; a value outside the fp16 range sends the chunk to the exact path
                {
                    const int r = warp * 16 + lane;
#pragma unroll
                    for (int c16 = 0; c16 < kNV / 16; ++c16) {
                        float u16[16];
                        tc::tmem_ld16(tmem + tl + kTmU + c16 * 16, u16);
                        tc::tmem_ld_wait();
                        if (lane < 16) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) bad |= !(fabsf(u16[i]) <= 65000.f);
                            *reinterpret_cast<uint4 *>(sm + SM::kUt + tile_chunk(r, 2 * c16, kChunk, kNV)) =
                                pack8_h(u16);
                            *reinterpret_cast<uint4 *>(sm + SM::kUt + tile_chunk(r, 2 * c16 + 1, kChunk, kNV)) =
                                pack8_h(u16 + 8);
                        }
                    }
                    tc::fence_async_smem();
                    tc::tc_fence_before();
                }
                bad = tc::named_sync_or(kBarChain, kChainThreads, bad);
                if (!role_wait(&full2, c & 1, leader, kBarChain, kChainThreads, &abort_flag)) break;
                part2_done = true;
                if (leader) tc::mbar_arrive_cluster(tc::mapa(tc::smem_u32(&consumed), prod));
                if (!bad) {
                    // ---- M4: O += P U~,  Sn = Kd^T U~ ----
                    if (leader) {
                        constexpr uint32_t idO = tc::make_idesc(64, kNV, tc::kF16, false, true);
                        constexpr uint32_t idS = tc::make_idesc(128, kNV, tc::kF16, true, true);
#pragma unroll
                        for (int kk = 0; kk < kChunk / 16; ++kk) {
                            const uint64_t bdesc = desc_mnmajor(sbase + SM::kUt, kChunk, kNV, kk);
                            tc::mma_f16(tmem + kTmO, desc_kmajor(sbase + SM::kSlot + I::kP, kChunk, kk), bdesc, idO,
                                        true);
                            tc::mma_f16(tmem + kTmSn, desc_mnmajor(sbase + SM::kSlot + I::kKd, kChunk, kDK, kk),
                                        bdesc, idS, kk > 0);
                        }
                        tc::mma_commit(&bar_m4);
                    }
                    if (!role_wait(&bar_m4, ph_m4, leader, kBarChain, kChainThreads, &abort_flag)) break;
                    ph_m4 ^= 1u;
                    if (leader && pre1) {
                        issue_part2(c + 1);
                        pre2 = true;
                    }
                    // ---- epilogue: output rows, state update ----
                    const int r = warp * 16 + lane;
                    float o[kNV], sn[kNV];
#pragma unroll
                    for (int c16 = 0; c16 < kNV / 16; ++c16) {
                        float x16[16];
                        tc::tmem_ld16(tmem + tl + kTmSn + c16 * 16, x16);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i) sn[c16 * 16 + i] = x16[i];
                        tc::tmem_ld16(tmem + tl + kTmO + c16 * 16, x16);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[c16 * 16 + i] = x16[i];
                    }
                    bool obad = false;
                    if (lane < 16)
#pragma unroll
                        for (int i = 0; i < kNV; ++i) obad |= !(fabsf(o[i]) <= 3.0e38f);
                    tc::tc_fence_before();
                    bad = tc::named_sync_or(kBarChain, kChainThreads, obad);
                    if (!bad) {
#pragma unroll
                        for (int j = 0; j < kNV; ++j) S[j] = fmaf(gam, S[j], sn[j]);
                        write_state_operand();
                        if (lane < 16 && r < L) {
                            TO *dst = out + ((tok0 + r) * H + h) * DV + vcol0;
#pragma unroll
                            for (int c16 = 0; c16 < kNV / 16; ++c16) store16<TO>(dst + c16 * 16, &o[c16 * 16]);
                        }
                        tc::named_sync(kBarChain, kChainThreads);
                        continue;
                    }
                }
            }
            // exact path: the chunk's decays exceed the rebasing range, or an fp16 value overflowed
            if (!part2_done) {
                if (!role_wait(&full2, c & 1, leader, kBarChain, kChainThreads, &abort_flag)) break;
                if (leader) tc::mbar_arrive_cluster(tc::mapa(tc::smem_u32(&consumed), prod));
            }
            exact_chunk(tok0, L);
            tc::tc_fence_before();
            tc::named_sync(kBarChain, kChainThreads);
        }
        if (final_state && abort_flag == 0) {
#pragma unroll
            for (int j = 0; j < kNV; ++j) final_state[state_base + j] = S[j];
        }
    } else {
        // ===================================== prep role ======================================
        const int tp = tid - kChainThreads;      // 0..255
        const bool leader = tp == 0;
        const int cg = tp & 15, tg = tp >> 4;    // 8 channels [8cg, 8cg+8), 4 tokens [4tg, 4tg+4)
        uint8_t *img = sm + SM::kImg;
        uint4 rg[4], rk[4], rq[4];
        float rb = 0.f;
        auto load_raw = [&](int c) {
            const int64_t tok0 = t0 + (int64_t)c * kChunk;
            const int L = static_cast<int>((t1 - tok0) < kChunk ? (t1 - tok0) : kChunk);
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                const int r = tg * 4 + rr;
                if (r < L) {
                    const int64_t off = ((tok0 + r) * H + h) * kDK + cg * 8;
                    rg[rr] = *reinterpret_cast<const uint4 *>(log_alpha + off);
                    rk[rr] = *reinterpret_cast<const uint4 *>(k + off);
                    rq[rr] = *reinterpret_cast<const uint4 *>(q + off);
                } else {
                    rg[rr] = rk[rr] = rq[rr] = make_uint4(0, 0, 0, 0);
                }
            }
            rb = (tp < kChunk && tp < L) ? __bfloat162float(beta[(tok0 + tp) * H + h]) : 0.f;
        };
        // store the finished image and announce it to every chain of the cluster
        auto publish = [&](int c) -> bool {
            bool ok = true;
            if (leader) {
                if (c >= CL) ok = tc::mbar_wait_cluster(&consumed, (c / CL - 1) & 1, &abort_flag);
                if (ok) {
                    tc::bulk_store_and_wait(ws_cluster + (size_t)rank * I::kStride, img, I::kBytes);
                    tc::fence_async_global();
                    for (int r = 0; r < CL; ++r) tc::mbar_arrive_cluster(tc::mapa(tc::smem_u32(&pub[rank]), r));
                }
            }
            return !tc::named_sync_or(kBarPrep, kPrepThreads, !ok);
        };
        uint32_t ph_m1 = 0, ph_m2 = 0;
        constexpr int ld = SM::kLd;
        float *sA = reinterpret_cast<float *>(sm + SM::kA32);
        float *sT = reinterpret_cast<float *>(sm + SM::kT32);
        float *sX = reinterpret_cast<float *>(sm + SM::kX32);
        int *img_flag = reinterpret_cast<int *>(img + I::kFlag);
        float *img_gamma = reinterpret_cast<float *>(img + I::kGamma);
        if (rank < nchunks) load_raw(rank);
        for (int c = rank; c < nchunks; c += CL) {
            // ---- decays (fp32 scan over the chunk, per channel) ----
            float G[4][8];
            {
                float run[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) run[i] = 0.f;
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    float g8[8];
                    unpack8(rg[rr], g8);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        run[i] += g8[i];
                        G[rr][i] = run[i];
                    }
                }
                // lanes 16-31 hold the odd token group of the warp's pair: add the even one's total
                const int w4 = warp - 4;
                float pair_tot[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float lower = __shfl_up_sync(0xffffffffu, run[i], 16);
                    const float add = (lane >= 16) ? lower : 0.f;
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) G[rr][i] += add;
                    pair_tot[i] = run[i] + add;  // lanes 16-31: total of the warp's 8 tokens
                }
                if (lane >= 16) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) sTot[w4 * kDK + cg * 8 + i] = pair_tot[i];
                }
                if (tp < kChunk) sBeta[tp] = rb;
                tc::named_sync(kBarPrep, kPrepThreads);
                float off[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) off[i] = 0.f;
                for (int pw = 0; pw < w4; ++pw)
#pragma unroll
                    for (int i = 0; i < 8; ++i) off[i] += sTot[pw * kDK + cg * 8 + i];
#pragma unroll
                for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                    for (int i = 0; i < 8; ++i) G[rr][i] += off[i];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (tg == 0) sG0[cg * 8 + i] = G[0][i];
                    if (tg == 7) sGref[cg * 8 + i] = G[3][i];
                    if (tg == 15) sGlast[cg * 8 + i] = G[3][i];
                }
            }
            tc::named_sync(kBarPrep, kPrepThreads);
            bool bad = false;
            if (tp < kDK) {
                const float g0 = sG0[tp], gr = sGref[tp], gl = sGlast[tp];
                bad = !((g0 - gr <= kRangeLimit) && (gr - gl <= kRangeLimit));
            }
            if (tc::named_sync_or(kBarPrep, kPrepThreads, bad)) {
                // decays too fast for the rebased products: every chain evaluates it exactly
                if (c + CL < nchunks) load_raw(c + CL);
                if (leader) *img_flag = 1;
                tc::fence_async_smem();
                tc::named_sync(kBarPrep, kPrepThreads);
                if (!publish(c)) break;
                continue;
            }

            // ---- rebased and decayed operands ----
            {
                float gref[8], erefabs[8], elast[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    gref[i] = sGref[cg * 8 + i];
                    erefabs[i] = fast_exp(gref[i]);                       // exp(Gref)
                    elast[i] = fast_exp(sGlast[cg * 8 + i] - gref[i]);   // exp(Glast - Gref)
                }
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const int r = tg * 4 + rr;
                    float kf[8], qf[8];
                    unpack8(rk[rr], kf);
                    unpack8(rq[rr], qf);
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
                    *reinterpret_cast<uint4 *>(img + I::kQg + off) = pack8_h(qg);
                    *reinterpret_cast<uint4 *>(img + I::kKd + off) = pack8_h(kd);
                }
            }
            // the raw registers are consumed: fetch this CTA's next chunk
            if (c + CL < nchunks) load_raw(c + CL);
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::named_sync(kBarPrep, kPrepThreads);

            // ---- M1: A_raw = Kr Kn^T,  P_raw = Qr Kn^T (two-term split); one commit, since the
            //          UT scratch below reuses the operands of both ----
            if (leader) {
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
                tc::mma_commit(&bar_m1);
            }
            if (!role_wait(&bar_m1, ph_m1, leader, kBarPrep, kPrepThreads, &abort_flag)) break;
            ph_m1 ^= 1u;

            // ---- A (fp32, beta-scaled, strict lower) and tril(P) (fp16, into the image) ----
            {
                const int r = (warp & 3) * 16 + lane;
                if (warp < 8) {
                    const float br = (lane < 16) ? sBeta[r] : 0.f;
#pragma unroll
                    for (int c16 = 0; c16 < 4; ++c16) {
                        float x16[16];
                        tc::tmem_ld16(tmem + tl + kTmA + c16 * 16, x16);
                        tc::tmem_ld_wait();
                        if (lane < 16) {
#pragma unroll
                            for (int i = 0; i < 16; i += 4)
                                *reinterpret_cast<float4 *>(&sA[r * ld + c16 * 16 + i]) =
                                    make_float4((c16 * 16 + i < r) ? br * x16[i] : 0.f,
                                                (c16 * 16 + i + 1 < r) ? br * x16[i + 1] : 0.f,
                                                (c16 * 16 + i + 2 < r) ? br * x16[i + 2] : 0.f,
                                                (c16 * 16 + i + 3 < r) ? br * x16[i + 3] : 0.f);
                        }
                    }
                } else {
#pragma unroll
                    for (int c16 = 0; c16 < 4; ++c16) {
                        float x16[16];
                        tc::tmem_ld16(tmem + tl + kTmP + c16 * 16, x16);
                        tc::tmem_ld_wait();
                        if (lane < 16) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) x16[i] = (c16 * 16 + i <= r) ? x16[i] : 0.f;
                            *reinterpret_cast<uint4 *>(img + I::kP + tile_chunk(r, 2 * c16, kChunk, kChunk)) =
                                pack8_h(x16);
                            *reinterpret_cast<uint4 *>(img + I::kP + tile_chunk(r, 2 * c16 + 1, kChunk, kChunk)) =
                                pack8_h(x16 + 8);
                        }
                    }
                }
            }
            tc::tc_fence_before();
            tc::named_sync(kBarPrep, kPrepThreads);

            // ---- UT transform T = (I + A)^{-1} ----
            // (a) 16x16 diagonal blocks: thread (bb, cc) solves column cc of (I + A_bb) x = e_cc by
            //     forward substitution; the zeros above the diagonal are written too.
            if (tp < 64) {
                const int bb = tp >> 4, cc = tp & 15;
                const float *arow = sA + (16 * bb) * ld + 16 * bb;
                float x[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < 15; ++s2)
                        if (s2 < r) {
                            const float term = arow[r * ld + s2] * ((s2 >= cc) ? x[s2] : 0.f);
                            if (s2 & 1) acc1 += term; else acc0 += term;
                        }
                    x[r] = (r == cc) ? 1.f : ((r > cc) ? -(acc0 + acc1) : 0.f);
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) sT[(16 * bb + r) * ld + 16 * bb + cc] = x[r];
            }
            tc::named_sync(kBarPrep, kPrepThreads);
            // (b) off-diagonal blocks by distance d = i - j: T_ij = -T_ii sum_{j<=m<i} A_im T_mj.
            //     The 4 - d blocks of one distance are independent; 256 threads = one 16x16 block.
#pragma unroll
            for (int d = 1; d < 4; ++d) {
                const int r = tp >> 4, cc = tp & 15;
#pragma unroll
                for (int blk = 0; blk < 4 - d; ++blk) {
                    const int j = blk, i = blk + d;
                    const float *arow = sA + (16 * i + r) * ld + 16 * j;
                    const float *tcol = sT + (16 * j) * ld + 16 * j + cc;
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int m = 0; m < 16 * d; m += 4) {
                        const float4 a4 = *reinterpret_cast<const float4 *>(arow + m);
                        acc[0] = fmaf(a4.x, tcol[(m + 0) * ld], acc[0]);
                        acc[1] = fmaf(a4.y, tcol[(m + 1) * ld], acc[1]);
                        acc[2] = fmaf(a4.z, tcol[(m + 2) * ld], acc[2]);
                        acc[3] = fmaf(a4.w, tcol[(m + 3) * ld], acc[3]);
                    }
                    sX[blk * 256 + r * 16 + cc] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
                }
                tc::named_sync(kBarPrep, kPrepThreads);
#pragma unroll
                for (int blk = 0; blk < 4 - d; ++blk) {
                    const int j = blk, i = blk + d;
                    const float *drow = sT + (16 * i + r) * ld + 16 * i;  // row r of T_ii (zero above the diagonal)
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int m = 0; m < 16; m += 4) {
                        const float4 t4 = *reinterpret_cast<const float4 *>(drow + m);
                        acc[0] = fmaf(t4.x, sX[blk * 256 + (m + 0) * 16 + cc], acc[0]);
                        acc[1] = fmaf(t4.y, sX[blk * 256 + (m + 1) * 16 + cc], acc[1]);
                        acc[2] = fmaf(t4.z, sX[blk * 256 + (m + 2) * 16 + cc], acc[2]);
                        acc[3] = fmaf(t4.w, sX[blk * 256 + (m + 3) * 16 + cc], acc[3]);
                    }
                    sT[(16 * i + r) * ld + 16 * j + cc] = -((acc[0] + acc[1]) + (acc[2] + acc[3]));
                }
                tc::named_sync(kBarPrep, kPrepThreads);
            }
            // T diag(beta) -> fp16 A operand [64 x 64] in the image: 2 chunks of 8 per thread; the
            // strictly upper blocks of sT are never written, so the mask j*8 + i <= r is applied here
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int idx = tp * 2 + e, r = idx >> 3, j = idx & 7;
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = (j * 8 + i <= r) ? sT[r * ld + j * 8 + i] * sBeta[j * 8 + i] : 0.f;
                *reinterpret_cast<uint4 *>(img + I::kTb + tile_chunk(r, j, kChunk, kChunk)) = pack8_h(f);
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::named_sync(kBarPrep, kPrepThreads);

            // ---- M2: W = (T b) Kg ----
            if (leader) {
                tc::tc_fence_after();
                constexpr uint32_t idW = tc::make_idesc(64, kDK, tc::kF16, false, true);
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk)
                    tc::mma_f16(tmem + kTmW, desc_kmajor(sbase + SM::kImg + I::kTb, kChunk, kk),
                                desc_mnmajor(sbase + SM::kKg, kChunk, kDK, kk), idW, kk > 0);
                tc::mma_commit(&bar_m2);
            }
            if (!role_wait(&bar_m2, ph_m2, leader, kBarPrep, kPrepThreads, &abort_flag)) break;
            ph_m2 ^= 1u;

            // ---- W -> fp16 A operand [64 x 128] in the image; gamma; flag ----
            {
                const int w4 = warp - 4;
                const int half = w4 >> 2;            // columns [64 half, 64 half + 64)
                const int r = (warp & 3) * 16 + lane;
#pragma unroll
                for (int c16 = 0; c16 < 4; ++c16) {
                    float w16[16];
                    tc::tmem_ld16(tmem + tl + kTmW + half * 64 + c16 * 16, w16);
                    tc::tmem_ld_wait();
                    if (lane < 16) {
                        const int j = half * 8 + 2 * c16;
                        *reinterpret_cast<uint4 *>(img + I::kW + tile_chunk(r, j, kChunk, kDK)) = pack8_h(w16);
                        *reinterpret_cast<uint4 *>(img + I::kW + tile_chunk(r, j + 1, kChunk, kDK)) =
                            pack8_h(w16 + 8);
                    }
                }
            }
            if (tp < kDK) img_gamma[tp] = fast_exp(sGlast[tp]);
            if (leader) *img_flag = 0;
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::named_sync(kBarPrep, kPrepThreads);
            if (!publish(c)) break;
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync();  // no CTA leaves while a peer may still signal its barriers
    if (warp == 0) tc::tmem_dealloc(tmem, kTmCols);
}

// Bytes of global workspace kda_chunk_fwd needs on the tensor-core path: one
// chunk image per (sequence, head, value slice).
inline size_t chunk_tc_workspace_bytes(int64_t pairs, int DV) {
    return static_cast<size_t>(pairs) * (DV / kNV) * ChunkImage::kStride;
}

template <int CL, typename TO>
cudaError_t launch_chunk_tc_cl(const void *q, const void *k, const void *v, const void *la, const void *beta,
                               const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H, int DV,
                               void *out, float *final_state, void *workspace, cudaStream_t stream) {
    auto kern = kda_chunk_tc_kernel<CL, TO>;
    const int smem = ChunkSmem::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int N = cu ? num_seqs : B;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(N) * H * CL);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16 *>(q),
                              static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v),
                              static_cast<const __nv_bfloat16 *>(la), static_cast<const __nv_bfloat16 *>(beta),
                              init_state, cu, num_seqs, T, H, DV, static_cast<TO *>(out), final_state,
                              static_cast<uint8_t *>(workspace));
}

template <typename TO>
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const void *la, const void *beta,
                            const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H, int DV,
                            void *out, float *final_state, void *workspace, cudaStream_t stream) {
    if (DV == 64)
        return launch_chunk_tc_cl<2, TO>(q, k, v, la, beta, init_state, cu, num_seqs, B, T, H, DV, out, final_state,
                                         workspace, stream);
    return launch_chunk_tc_cl<4, TO>(q, k, v, la, beta, init_state, cu, num_seqs, B, T, H, DV, out, final_state,
                                     workspace, stream);
}

}  // namespace kda
