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
// Work split.  Only U~ and the state update sit on the sequential chain; every
// other quantity depends on the chunk's own inputs alone.  One cluster of
// 1 + kNP CTAs handles one (sequence, head):
//   * prep CTAs (ranks 1..kNP): CTA 1 + p prepares chunks c = p mod kNP: decays,
//     rebased operands, A and P, the UT transform, then W and U on the tensor
//     cores.  The finished chunk image (-W, U, Qg = Q exp(G), Kd = K exp(G_last - G),
//     P, gamma = exp(G_last) and a flag) is bulk-stored to this producer's region
//     of a global workspace (it stays in L2) and announced to the chain CTA
//     through a remote mbarrier arrive;
//   * the chain CTA (rank 0) bulk-loads each image into a two-deep shared-memory
//     ring and runs, per chunk, one MMA group [-W ; Qg] S (rows 0-63 give
//     U~ - U, rows 64-127 give Qg S), the U~ epilogue, the MMAs Kd^T U~ and
//     [. ; P] U~ (adding P U~ to rows 64-127) and the fp32 state update, while
//     dedicated warps store the output rows.
// The chain CTA computes all d_v columns of S at once: a tcgen05.mma costs about
// the same for N = 32 and N = 128 value columns, so slicing d_v across CTAs would
// multiply the tensor-core time of the chain without shortening it.
//
// Precision (fp32 accumulation in TMEM, fp32 master state in registers, fp32
// decays and substitution, fp32 or bf16 output):
//   * A and P need the rebased factors below, whose range exceeds fp16: they are
//     bf16 operands, and P (which feeds the output directly) uses a two-term
//     bf16 split of both operands (hi*hi + hi*lo + lo*hi), ~16-bit accuracy.
//   * Every other product has operands bounded by the inputs and runs on fp16
//     operands (11-bit significand, same tensor rate as bf16).  A value outside
//     the fp16 range turns U~ or O non-finite; that is detected and the chunk is
//     recomputed on the exact path below.
//
// Exponent range ("log-domain accumulation", section 3 of "Designing and
// Deploying Hybrid MLA and Linear Attention Architectures for LLMs"): the
// products of A and P are formed as (k exp(G - G_ref)) . (k exp(G_ref - G))
// with G_ref the cumulative decay at the chunk's middle token, so each factor
// stays within exp(+-kRangeLimit) whenever the chunk's per-channel decay on
// either side of the middle stays within kRangeLimit.  A chunk whose decays
// exceed that (extremely fast forgetting) is evaluated token by token in fp32
// by the chain CTA instead, so every input with finite log_alpha gets a correct
// result.
//
// Packed variable-length batches are scheduled longest-first.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

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

constexpr int kNP = 3;                // prep CTAs per cluster
constexpr int kCL = kNP + 1;          // cluster: chain CTA (rank 0) + prep CTAs
constexpr int kRoleWarps = 16;                        // warps 0-15 run the role
constexpr int kRoleThreads = kRoleWarps * 32;
constexpr int kThreads = kRoleThreads + 64;           // + two helper warps that move data
constexpr uint32_t kBarRole = 1, kBarU = 2, kBarOut = 3;  // named barriers: warps 0-7, U~ warps, output warps

// ---- chunk image in the global workspace (fp16 tiles in their shared-memory layouts) ----------
template <int DV> struct Img {
    static constexpr int kNW = 0;                          // -W  [64 x 128]
    static constexpr int kUT = kNW + kChunk * kDK * 2;     // U^T [DV x 64]
    static constexpr int kQt = kUT + kChunk * DV * 2;      // Qg  [64 x 128]
    static constexpr int kKd = kQt + kChunk * kDK * 2;     // Kd  [64 x 128]
    static constexpr int kP = kKd + kChunk * kDK * 2;      // tril(P) [64 x 64] (after Kd: [Kd ; P] rows)
    static constexpr int kGam = kP + kChunk * kChunk * 2;  // fp32 [128] exp(G_last)
    static constexpr int kFlag = kGam + kDK * 4;           // int: 1 = evaluate exactly
    static constexpr int kBytes = kFlag + 16;
    static constexpr int kStride = (kBytes + 1023) / 1024 * 1024;
};

// ---- chain CTA shared memory ------------------------------------------------------------------
template <int DV> struct ChainSmem {
    using I = Img<DV>;
    // one slot of the image ring: A1 = [-W ; Qg] as two 16 KB k-blocks of 128 rows (rows 0-63 -W,
    // rows 64-127 Qg; the B operand of S^T A1^T), then U^T, then Kd, P, gamma, flag in image order
    static constexpr int kA1 = 0;
    static constexpr int kUT = 2 * kChunk * kDK * 2;
    static constexpr int kKd = kUT + kChunk * DV * 2;
    static constexpr int kP = kKd + (I::kP - I::kKd);
    static constexpr int kGam = kKd + (I::kGam - I::kKd);
    static constexpr int kFlag = kKd + (I::kFlag - I::kKd);
    static constexpr int kTailBytes = I::kBytes - I::kKd;
    static constexpr int kSlotBytes = (kKd + kTailBytes + 1023) / 1024 * 1024;
    // exact path scratch (fp32): per-column partial sums of S^T k and S^T q per channel quarter, k . q
    static constexpr int kRedPk = 2 * kSlotBytes;
    static constexpr int kRedPq = kRedPk + 4 * 128 * 4;
    static constexpr int kRedKq = kRedPq + 4 * 128 * 4;
    // output staging of a full chunk: DV / 64 blocks of [64 tokens x 64 values] (fp32 or bf16),
    // written by a TMA tensor store per block
    static constexpr int kOut = (kRedKq + 16 + 1023) / 1024 * 1024;
    static constexpr int kBytes = kOut + kChunk * DV * 4;
};

// ---- prep CTA shared memory -------------------------------------------------------------------
template <int DV> struct PrepSmem {
    using I = Img<DV>;
    static constexpr int kTile = kChunk * kDK * 2;         // [64 x 128] 16-bit tile
    // A operands of the A/P products, per 64-channel block b: [Kr_b | Qh_b | Ql_b]
    // (8 KB each), so that [Kr ; Qh] and [Qh ; Ql] are 128-row operands
    static constexpr int kKQBlk = 3 * kChunk * 128;
    static constexpr int kKQ = 0;
    static constexpr int kKh = 2 * kKQBlk;                 // K exp(Gref - G), hi  [64 x 128] (B)
    static constexpr int kKl = kKh + kTile;                //                  lo
    static constexpr int kKgV = kKl + kTile;               // [K exp(G) | V] [64 x 256], V zero past DV
    // [Tb | Tb]: the A operand of W (both row halves give the same rows, so all warps can read
    // them); the first Tb is also the B operand of U^T = V^T Tb^T
    static constexpr int kTbP = kKgV + kChunk * 2 * kDK * 2;
    static constexpr int kImg = kTbP + 2 * kChunk * kChunk * 2;  // staging image (Img layout)
    static constexpr int kBeta = kImg + I::kStride;              // fp32 [64]
    static constexpr int kG0 = kBeta + kChunk * 4;               // fp32 [128] decay after token 0
    static constexpr int kGref = kG0 + kDK * 4;                  //            after token 31
    static constexpr int kGlast = kGref + kDK * 4;               //            after token 63
    static constexpr int kBytes = kGlast + kDK * 4;
    // The A/P operand area also holds, in turn: the raw bf16 inputs of the chunk (bulk-loaded
    // rows of log_alpha, k, q, v; read into registers before the operands are written) and the
    // fp32 scratch of the UT transform (once the A/P products complete).
    static constexpr int kRawG = 0, kRawK = kChunk * 256, kRawQ = 2 * kChunk * 256, kRawV = 3 * kChunk * 256;
    static constexpr int kRawBytes = kChunk * (3 * kDK * 2 + DV * 2);   // one TMA box per tensor
    static constexpr int kLd = 68;                               // row stride of A and T^T
    static constexpr int kA32 = 0;                               // A [64][68]
    static constexpr int kT32 = kA32 + kChunk * kLd * 4;         // T^T [64][68] (row c = column c of T)
    static constexpr int kX32 = kT32 + kChunk * kLd * 4;         // [3][16][20] block products, transposed
    static constexpr int kTd32 = kX32 + 3 * 16 * 20 * 4;         // [4][16][20] diagonal blocks of T
    static_assert(kTd32 + 4 * 16 * 20 * 4 <= kKgV && kRawV + kChunk * DV * 2 <= kKgV, "A/P operand area");
    // scan scratch inside the K exp(G) | V operand (dead from [W | U] to the next rebase)
    static constexpr int kTot = kKgV;                            // [16][128] per-warp totals
    static constexpr int kPre = kTot + 16 * kDK * 4;             // [16][128] per-warp prefixes
};

template <int DV> constexpr int chunk_smem_bytes() {
    return (ChainSmem<DV>::kBytes > PrepSmem<DV>::kBytes ? ChainSmem<DV>::kBytes : PrepSmem<DV>::kBytes) + 1024;
}
static_assert(chunk_smem_bytes<128>() <= 232448, "shared memory plan exceeds 227 KB");

// TMEM columns (fp32 accumulators, M = 128 layout: row m -> lane m).
// chain: D1^T double-buffered (0, 128), D2^T, the S^T operand (64 columns) and the U~^T operand (32)
constexpr uint32_t kTmD1 = 0, kTmD2 = 256, kTmS = 384, kTmUt = 448, kTmChainCols = 512;
constexpr uint32_t kTmA = 0, kTmP2 = 64, kTmW = 256, kTmUT = 384, kTmPrepCols = 512;  // prep

// Descriptor of k-step `kk` (16 elements along K) of a K-major SW128 operand with `rows` rows.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int rows, int kk) {
    return tc::make_sdesc(base + (kk >> 2) * (rows * 128) + (kk & 3) * 32, 16, 1024, tc::kSwz128);
}
// Descriptor of k-step `kk` of an MN-major operand stored as [K rows x MN columns] in 64-column
// SW128 blocks of krows x 128 bytes.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, int krows, int kk) {
    return tc::make_sdesc(base + kk * 2048, krows * 128, 1024, tc::kSwz128);
}
// Byte offset of 16-byte chunk `j` (8 16-bit columns) of row `r` in a tile with `rows` rows
// stored as 64-column SW128 blocks.
__device__ __forceinline__ uint32_t tile_chunk(int r, int j, int rows) {
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
__device__ __forceinline__ void unpack8_h(const uint4 &u, float *f) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 x = __half22float2(h[i]);
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
// Same with a phase completed by other CTAs of the cluster.
__device__ __forceinline__ bool role_wait_cluster(uint64_t *bar, uint32_t parity, bool leader, uint32_t bar_id,
                                                  uint32_t nthreads, volatile int *abort_flag) {
    bool ok = true;
    if (leader) ok = tc::mbar_wait_cluster(bar, parity, abort_flag);
    const bool failed = tc::named_sync_or(bar_id, nthreads, !ok);
    tc::tc_fence_after();
    return !failed;
}

// Wait (bounded, ignoring the abort flag) for all tcgen05 operations this thread issued.
__device__ __forceinline__ void drain_mma(uint64_t *bar, uint32_t parity) {
    int never = 0;
    tc::mma_commit(bar);
    tc::mbar_wait(bar, parity, &never);
}

// Per-CTA bookkeeping shared by both roles.
struct ChunkCtx {
    int n, h, H, nchunks;
    int64_t t0, t1;
    uint32_t sbase, tmem;
    uint8_t *sm;
    uint8_t *ws_pair;        // this (sequence, head)'s kNP producer regions
    volatile int *abort_flag;
    // chunk c: first token and valid length
    __device__ __forceinline__ int64_t tok0(int c) const { return t0 + (int64_t)c * kChunk; }
    __device__ __forceinline__ int len(int c) const {
        const int64_t r = t1 - tok0(c);
        return static_cast<int>(r < kChunk ? r : kChunk);
    }
};

// Mbarriers of one CTA (each role uses its own subset).
struct ChunkBars {
    // chain: image slot full / free, MMA completions, producer publications (per producer region)
    uint64_t full[2], slot_free[2], mma1, mma2, mma3[2], pub[kNP][2];
    // prep: MMA completions, global region consumed by the chain (per region)
    uint64_t m_ap, m_wu, consumed[2], staged, staging_free, raw_full, raw_free;
    uint64_t fin;
    int chain_ok;   // the chain leader's last MMA wait succeeded (read after a barrier)
};

// Tensor maps of the token tensors: [tokens][H][d] bf16, one box = 64 tokens x d channels of one
// head; and of the output [tokens][H][d_v] (fp32 or bf16), one box = 64 tokens x 64 values.
struct RowMaps {
    CUtensorMap g, k, q, v, o;
};

// ================================== prep role (cluster ranks 1..kNP) ==================================
// Producer p prepares chunks c = p, p + kNP, ... with warps 0-15.  Lane 0 of warp 16 stores each
// finished image to one of the producer's two global regions and announces it; lane 0 of warp 17
// loads the raw input tiles of the next chunk.
template <int DV>
__device__ __forceinline__ void prep_role(const ChunkCtx &cx, ChunkBars &bars, int p, const RowMaps &maps,
                                          const __nv_bfloat16 *beta) {
    using SM = PrepSmem<DV>;
    using I = Img<DV>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t *const sm = cx.sm;
    const uint32_t sbase = cx.sbase, tmem = cx.tmem;
    const int H = cx.H, h = cx.h, nchunks = cx.nchunks;
    volatile int *abort_flag = cx.abort_flag;
    if (warp == kRoleWarps) {
        if (lane == 0) {
            // ---- publisher: staged image -> the chunk's global region (one bulk store), then announce
            //      the region to the chain CTA ----
            int kl = 0;
            for (int c = p; c < nchunks; c += kNP, ++kl) {
                const int reg = kl & 1;
                uint8_t *gimg = cx.ws_pair + (size_t)(p * 2 + reg) * I::kStride;
                if (!tc::mbar_wait(&bars.staged, kl & 1, abort_flag)) break;
                tc::bulk_store_nc(gimg, sm + SM::kImg, I::kBytes);
                tc::bulk_commit();
                tc::bulk_wait_read_all();
                tc::mbar_arrive(&bars.staging_free);
                tc::bulk_wait_all();
                tc::fence_async_global();
                tc::mbar_arrive_cluster(tc::mapa(tc::smem_u32(&bars.pub[p][reg]), 0));
            }
        }
        return;
    }
    if (warp == kRoleWarps + 1) {
        if (lane == 0) {
            // ---- raw input loader: the 64-token tiles of log_alpha, k, q, v of this producer's next
            //      chunk (TMA; rows past the tensor end read as zero, rows past the sequence end are
            //      masked by the readers), into the A/P operand area once the previous chunk's UT
            //      scratch is dead ----
            int kl = 0, issued = -1;
            for (int c = p; c < nchunks; c += kNP, ++kl) {
                if (kl >= 1 && !tc::mbar_wait(&bars.raw_free, (kl - 1) & 1, abort_flag)) break;
                const int t = static_cast<int>(cx.tok0(c));
                tc::mbar_arrive_expect_tx(&bars.raw_full, SM::kRawBytes);
                tc::tma_load_3d(sm + SM::kRawG, &maps.g, 0, h, t, &bars.raw_full);
                tc::tma_load_3d(sm + SM::kRawK, &maps.k, 0, h, t, &bars.raw_full);
                tc::tma_load_3d(sm + SM::kRawQ, &maps.q, 0, h, t, &bars.raw_full);
                tc::tma_load_3d(sm + SM::kRawV, &maps.v, 0, h, t, &bars.raw_full);
                issued = kl;
            }
            // no copy may still be in flight when the CTA leaves
            if (issued >= 0) {
                int never = 0;
                tc::mbar_wait(&bars.raw_full, issued & 1, &never);
            }
        }
        return;
    }

    // ---- compute warps 0-15 ----
    const int tp = tid;
    const bool leader = tp == 0;
    const int cg = tp & 15, tg = tp >> 4;   // channels [8cg, 8cg+8), tokens 2tg, 2tg + 1
    const int sp = warp & 3, q4 = warp >> 2;
    const uint32_t tl = tc::tmem_lane_base(warp);
    float *sBeta = reinterpret_cast<float *>(sm + SM::kBeta);
    float *sG0 = reinterpret_cast<float *>(sm + SM::kG0);
    float *sGref = reinterpret_cast<float *>(sm + SM::kGref);
    float *sGlast = reinterpret_cast<float *>(sm + SM::kGlast);
    float *sTot = reinterpret_cast<float *>(sm + SM::kTot);
    float *sPre = reinterpret_cast<float *>(sm + SM::kPre);
    constexpr int ld = SM::kLd;
    float *sA = reinterpret_cast<float *>(sm + SM::kA32);
    float *sT = reinterpret_cast<float *>(sm + SM::kT32);
    float *sX = reinterpret_cast<float *>(sm + SM::kX32);
    float *sTd = reinterpret_cast<float *>(sm + SM::kTd32);

    // beta of the next chunk, prefetched into registers (one value per thread of warps 0-1)
    float rb = 0.f;
    auto load_beta = [&](int c) {
        const int64_t tok0 = cx.tok0(c);
        rb = (tp < kChunk && tp < cx.len(c)) ? __bfloat162float(beta[(tok0 + tp) * H + h]) : 0.f;
    };
    // the staged chunk image is complete: set its flag (1: some value left the fp16 range, or the
    // decays the rebasing range; the chain then evaluates the chunk exactly) and hand it to the
    // publisher
    uint8_t *const img = sm + SM::kImg;
    auto stage_done = [&](bool mybad) {
        tc::fence_async_smem();
        const bool bad = tc::named_sync_or(kBarRole, kRoleThreads, mybad);
        if (leader) {
            *reinterpret_cast<volatile int *>(img + I::kFlag) = bad ? 1 : 0;
            tc::fence_async_smem();
            tc::mbar_arrive(&bars.staged);
        }
    };

    uint32_t ph_ap = 0, ph_wu = 0;
    if (p < nchunks) load_beta(p);
    int kl = 0;
    for (int c = p; c < nchunks; c += kNP, ++kl) {
        const int reg = kl & 1;
        // region `reg` last held this producer's chunk kl - 2: the chain must have loaded it
        if (kl >= 2 &&
            !role_wait_cluster(&bars.consumed[reg], ((kl >> 1) - 1) & 1, leader, kBarRole, kRoleThreads, abort_flag))
            break;
        const int L = cx.len(c);
        // the raw inputs of this chunk are in shared memory
        if (!role_wait(&bars.raw_full, kl & 1, leader, kBarRole, kRoleThreads, abort_flag)) break;
        // ---- decays: fp32 scan over the chunk, per channel ----
        float G[2][8];
        {
            float run[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) run[i] = 0.f;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = tg * 2 + rr;
                float g8[8];
                const uint4 raw = r < L ? *reinterpret_cast<const uint4 *>(sm + SM::kRawG + r * 256 + cg * 16)
                                        : make_uint4(0, 0, 0, 0);
                unpack8(raw, g8);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    run[i] += g8[i];
                    G[rr][i] = run[i];
                }
            }
            // lanes 16-31 hold the later token pair of the warp's four tokens: add the earlier total
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float lower = __shfl_up_sync(0xffffffffu, run[i], 16);
                const float add = (lane >= 16) ? lower : 0.f;
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) G[rr][i] += add;
                if (lane >= 16) sTot[warp * kDK + cg * 8 + i] = run[i] + add;   // the warp's 4 tokens
            }
            if (tg == 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) sG0[cg * 8 + i] = G[0][i];             // token 0: no prefix
            }
            if (tp < kChunk) sBeta[tp] = rb;
        }
        tc::named_sync(kBarRole, kRoleThreads);
        // per channel: exclusive prefix over the 16 warps, G after tokens 31 and 63, range check
        bool bad = false;
        if (tp < kDK) {
            float run = 0.f, gref = 0.f;
#pragma unroll
            for (int w = 0; w < kRoleWarps; ++w) {
                sPre[w * kDK + tp] = run;
                run += sTot[w * kDK + tp];
                if (w == 7) gref = run;
            }
            sGref[tp] = gref;
            sGlast[tp] = run;
            bad = !((sG0[tp] - gref <= kRangeLimit) && (gref - run <= kRangeLimit));
        }
        if (tc::named_sync_or(kBarRole, kRoleThreads, bad)) {
            // decays too fast for the rebased products: the chain evaluates this chunk exactly
            if (c + kNP < nchunks) load_beta(c + kNP);
            if (leader) tc::mbar_arrive(&bars.raw_free);
            if (kl >= 1 &&
                !role_wait(&bars.staging_free, (kl - 1) & 1, leader, kBarRole, kRoleThreads, abort_flag))
                break;
            stage_done(true);
            continue;
        }
        {
            float off[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) off[i] = sPre[warp * kDK + cg * 8 + i];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                for (int i = 0; i < 8; ++i) G[rr][i] += off[i];
        }

        // the publisher has read the previous image out of the staging tiles
        if (kl >= 1 &&
            !role_wait(&bars.staging_free, (kl - 1) & 1, leader, kBarRole, kRoleThreads, abort_flag))
            break;
        // ---- rebased and decayed operands; Q exp(G) and Kd into the staged image ----
        bool ovf = false;   // an fp16 operand or image value out of range
        uint4 rk[2], rq[2], rv[2];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int r = tg * 2 + rr;
            const bool in = r < L;
            rk[rr] = in ? *reinterpret_cast<const uint4 *>(sm + SM::kRawK + r * 256 + cg * 16) : make_uint4(0, 0, 0, 0);
            rq[rr] = in ? *reinterpret_cast<const uint4 *>(sm + SM::kRawQ + r * 256 + cg * 16) : make_uint4(0, 0, 0, 0);
            rv[rr] = (in && cg * 8 < DV) ? *reinterpret_cast<const uint4 *>(sm + SM::kRawV + r * DV * 2 + cg * 16)
                                         : make_uint4(0, 0, 0, 0);
        }
        tc::named_sync(kBarRole, kRoleThreads);   // the operands below overwrite the raw rows
        {
            float gref[8], elast[8], erefabs[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                gref[i] = sGref[cg * 8 + i];
                erefabs[i] = fast_exp(gref[i]);                       // exp(Gref)
                elast[i] = fast_exp(sGlast[cg * 8 + i] - gref[i]);   // exp(Glast - Gref)
            }
            const uint32_t okq = SM::kKQ + (cg >> 3) * SM::kKQBlk;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = tg * 2 + rr;
                float kf[8], qf[8];
                unpack8(rk[rr], kf);
                unpack8(rq[rr], qf);
                float kr[8], qr[8], kn[8], kd[8], kg[8], qg[8], vf[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float dg = G[rr][i] - gref[i];
                    const float e1 = fast_exp(dg), e2 = fast_exp(-dg);
                    kr[i] = kf[i] * e1;
                    qr[i] = qf[i] * e1;
                    kn[i] = kf[i] * e2;
                    kd[i] = kn[i] * elast[i];
                    kg[i] = kr[i] * erefabs[i];
                    qg[i] = qr[i] * erefabs[i];
                }
                const uint32_t o128 = tile_chunk(r, cg, kChunk);   // [64 x 128] tiles
                *reinterpret_cast<uint4 *>(sm + SM::kKgV + o128) = pack8_h(kg);
                *reinterpret_cast<uint4 *>(img + I::kQt + o128) = pack8_h(qg);
                unpack8(rv[rr], vf);   // zero past DV
#pragma unroll
                for (int i = 0; i < 8; ++i) ovf |= !(fabsf(vf[i]) <= 65000.f);
                *reinterpret_cast<uint4 *>(sm + SM::kKgV + tile_chunk(r, 16 + cg, kChunk)) = pack8_h(vf);
                const uint32_t okr = okq + tc::sw128(r, cg & 7);   // [Kr | Qh | Ql] blocks
                uint4 hi, lo;
                *reinterpret_cast<uint4 *>(sm + okr) = pack8_bf16(kr);
                split8_bf16(qr, hi, lo);
                *reinterpret_cast<uint4 *>(sm + okr + 8192) = hi;
                *reinterpret_cast<uint4 *>(sm + okr + 16384) = lo;
                split8_bf16(kn, hi, lo);
                *reinterpret_cast<uint4 *>(sm + SM::kKh + o128) = hi;
                *reinterpret_cast<uint4 *>(sm + SM::kKl + o128) = lo;
                *reinterpret_cast<uint4 *>(img + I::kKd + o128) = pack8_h(kd);
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        tc::named_sync(kBarRole, kRoleThreads);

        // ---- A/P products: D_A = [Kr ; Qh] Kh^T (rows 0-63 A_raw, rows 64-127 Qh Kh^T),
        //      D_P2 = [Kr ; Qh] Kl^T + [Qh ; Ql] Kh^T (rows 64-127 Qh Kl^T + Ql Kh^T) ----
        if (leader) {
            tc::tc_fence_after();
            constexpr uint32_t id = tc::make_idesc(128, 64, tc::kBF16, false, false);
#pragma unroll
            for (int kk = 0; kk < kDK / 16; ++kk) {
                const uint32_t a0 = sbase + SM::kKQ + (kk >> 2) * SM::kKQBlk + (kk & 3) * 32;
                const uint64_t akq = tc::make_sdesc(a0, 16, 1024, tc::kSwz128);
                const uint64_t aqq = tc::make_sdesc(a0 + 8192, 16, 1024, tc::kSwz128);
                const uint64_t bh = desc_kmajor(sbase + SM::kKh, kChunk, kk);
                const uint64_t bl = desc_kmajor(sbase + SM::kKl, kChunk, kk);
                tc::mma_f16(tmem + kTmA, akq, bh, id, kk > 0);
                tc::mma_f16(tmem + kTmP2, akq, bl, id, kk > 0);
                tc::mma_f16(tmem + kTmP2, aqq, bh, id, true);
            }
            tc::mma_commit(&bars.m_ap);
        }
        if (c + kNP < nchunks) load_beta(c + kNP);
        if (!role_wait(&bars.m_ap, ph_ap, leader, kBarRole, kRoleThreads, abort_flag)) break;
        ph_ap ^= 1u;

        // ---- A (fp32, beta-scaled, strict lower) and tril(P) (fp16, into the image): warp (sp, q4)
        //      reads accumulator rows 32 sp + lane, columns 16 q4 + [0, 16) ----
        {
            const int m = sp * 32 + lane;
            const int cb = q4 * 16;
            float x16[16];
            tc::tmem_ld16(tmem + tl + kTmA + cb, x16);
            if (sp < 2) {
                tc::tmem_ld_wait();
                const int r = m;
                const float br = sBeta[r];
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4 *>(&sA[r * ld + cb + i]) =
                        make_float4((cb + i < r) ? br * x16[i] : 0.f, (cb + i + 1 < r) ? br * x16[i + 1] : 0.f,
                                    (cb + i + 2 < r) ? br * x16[i + 2] : 0.f,
                                    (cb + i + 3 < r) ? br * x16[i + 3] : 0.f);
            } else {
                float y16[16];
                tc::tmem_ld16(tmem + tl + kTmP2 + cb, y16);
                tc::tmem_ld_wait();
                const int r = m - 64;
#pragma unroll
                for (int i = 0; i < 16; ++i) x16[i] = (cb + i <= r) ? x16[i] + y16[i] : 0.f;
                *reinterpret_cast<uint4 *>(img + I::kP + tile_chunk(r, cb / 8, kChunk)) = pack8_h(x16);
                *reinterpret_cast<uint4 *>(img + I::kP + tile_chunk(r, cb / 8 + 1, kChunk)) = pack8_h(x16 + 8);
            }
        }
        tc::tc_fence_before();
        tc::named_sync(kBarRole, kRoleThreads);

        // ---- UT transform T = (I + A)^{-1}, stored transposed (sT row c = column c of T) ----
        // (a) 16x16 diagonal blocks: eight threads (pp = tp % 8) solve column cc of (I + A_bb) x = e_cc
        //     by right-looking substitution: thread pp keeps rows pp and pp + 8 in registers, the
        //     owner of row s finalises x_s and shuffles it to the others, which update their later
        //     rows.  The zeros above the diagonal are written too.
        {
            const int col = tp >> 3, pp = tp & 7;
            const int bb = col >> 4, cc = col & 15;
            float a[2][16], part[2], x[2];
#pragma unroll
            for (int kq = 0; kq < 2; ++kq) {
                const float *arow = sA + (16 * bb + pp + 8 * kq) * ld + 16 * bb;
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const float4 v4 = *reinterpret_cast<const float4 *>(arow + 4 * s4);
                    a[kq][4 * s4] = v4.x;
                    a[kq][4 * s4 + 1] = v4.y;
                    a[kq][4 * s4 + 2] = v4.z;
                    a[kq][4 * s4 + 3] = v4.w;
                }
                part[kq] = 0.f;
            }
#pragma unroll
            for (int s2 = 0; s2 < 16; ++s2) {
                float xs = (s2 == cc) ? 1.f : ((s2 < cc) ? 0.f : -part[s2 >> 3]);
                xs = __shfl_sync(0xffffffffu, xs, (lane & ~7) | (s2 & 7));
                if (pp == (s2 & 7)) x[s2 >> 3] = xs;
#pragma unroll
                for (int kq = 0; kq < 2; ++kq)
                    if (pp + 8 * kq > s2) part[kq] = fmaf(a[kq][s2], xs, part[kq]);
            }
#pragma unroll
            for (int kq = 0; kq < 2; ++kq) {
                sT[(16 * bb + cc) * ld + 16 * bb + pp + 8 * kq] = x[kq];   // T^T
                sTd[(bb * 16 + pp + 8 * kq) * 20 + cc] = x[kq];            // T_bb, row-major
            }
        }
        tc::named_sync(kBarRole, kRoleThreads);
        // (b) off-diagonal blocks by distance d = i - j: T_ij = -T_ii sum_{j<=m<i} A_im T_mj.
        //     The 4 - d blocks of one distance are independent: entry e = blk * 256 + r * 16 + cc,
        //     threads take e = tp and tp + 512.  With T stored transposed, both factors of every dot
        //     product are contiguous (float4 reads).
#pragma unroll 1
        for (int d = 1; d < 4; ++d) {
            const int ne = (4 - d) * 256;
#pragma unroll 1
            for (int e = tp; e < ne; e += kRoleThreads) {
                const int blk = e >> 8, r = (e >> 4) & 15, cc = e & 15;
                const int j = blk, i = blk + d;
                const float *arow = sA + (16 * i + r) * ld + 16 * j;     // A[16i + r][16j + m]
                const float *tcol = sT + (16 * j + cc) * ld + 16 * j;    // T[16j + m][16j + cc]
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                for (int m = 0; m < 16 * d; m += 4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(arow + m);
                    const float4 t4 = *reinterpret_cast<const float4 *>(tcol + m);
                    acc[0] = fmaf(a4.x, t4.x, acc[0]);
                    acc[1] = fmaf(a4.y, t4.y, acc[1]);
                    acc[2] = fmaf(a4.z, t4.z, acc[2]);
                    acc[3] = fmaf(a4.w, t4.w, acc[3]);
                }
                sX[(blk * 16 + cc) * 20 + r] = (acc[0] + acc[1]) + (acc[2] + acc[3]);   // X^T
            }
            tc::named_sync(kBarRole, kRoleThreads);
#pragma unroll 1
            for (int e = tp; e < ne; e += kRoleThreads) {
                const int blk = e >> 8, r = (e >> 4) & 15, cc = e & 15;
                const int j = blk, i = blk + d;
                const float *drow = sTd + (i * 16 + r) * 20;   // T_ii[r][m] (zero above the diagonal)
                const float *xcol = sX + (blk * 16 + cc) * 20;  // X[m][cc]
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 16; m += 4) {
                    const float4 t4 = *reinterpret_cast<const float4 *>(drow + m);
                    const float4 x4 = *reinterpret_cast<const float4 *>(xcol + m);
                    acc[0] = fmaf(t4.x, x4.x, acc[0]);
                    acc[1] = fmaf(t4.y, x4.y, acc[1]);
                    acc[2] = fmaf(t4.z, x4.z, acc[2]);
                    acc[3] = fmaf(t4.w, x4.w, acc[3]);
                }
                sT[(16 * j + cc) * ld + 16 * i + r] = -((acc[0] + acc[1]) + (acc[2] + acc[3]));   // T^T
            }
            tc::named_sync(kBarRole, kRoleThreads);
        }
        // T diag(beta) -> fp16 A operand [64 x 64], one chunk of 8 per thread; the strictly upper
        // blocks of T are never written, so the mask s <= r is applied here
        {
            const int r = tp >> 3, j = tp & 7;
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = (j * 8 + i <= r) ? sT[(j * 8 + i) * ld + r] * sBeta[j * 8 + i] : 0.f;
            const uint4 t8 = pack8_h(f);
            *reinterpret_cast<uint4 *>(sm + SM::kTbP + tile_chunk(r, j, kChunk)) = t8;
            *reinterpret_cast<uint4 *>(sm + SM::kTbP + 8192 + tile_chunk(r, j, kChunk)) = t8;
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        tc::named_sync(kBarRole, kRoleThreads);
        if (leader) tc::mbar_arrive(&bars.raw_free);   // the UT scratch is dead: next raw rows may land

        // ---- W = Tb Kg, twice (A = [Tb ; Tb]);  U^T = V^T Tb^T (A = V^T, MN-major; B = Tb) ----
        if (leader) {
            tc::tc_fence_after();
            constexpr uint32_t idW = tc::make_idesc(128, kDK, tc::kF16, false, true);
            constexpr uint32_t idUT = tc::make_idesc(128, kChunk, tc::kF16, true, false);
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk) {
                tc::mma_f16(tmem + kTmW, tc::make_sdesc(sbase + SM::kTbP + kk * 32, 16, 1024, tc::kSwz128),
                            desc_mnmajor(sbase + SM::kKgV, kChunk, kk), idW, kk > 0);
                tc::mma_f16(tmem + kTmUT, desc_mnmajor(sbase + SM::kKgV + 2 * 8192, kChunk, kk),
                            desc_kmajor(sbase + SM::kTbP, kChunk, kk), idUT, kk > 0);
            }
            tc::mma_commit(&bars.m_wu);
        }
        if (tp < kDK) reinterpret_cast<float *>(img + I::kGam)[tp] = fast_exp(sGlast[tp]);
        if (!role_wait(&bars.m_wu, ph_wu, leader, kBarRole, kRoleThreads, abort_flag)) break;
        ph_wu ^= 1u;
        // -W (rows 0-63, duplicated in 64-127: warp (sp, q4) takes rows 32 (sp % 2) + lane, columns
        // 64 (sp / 2) + 16 q4 + [0, 16)) and U^T (value row j = 32 sp + lane, tokens 16 q4 + [0, 16))
        // -> fp16 in the staged image
        {
            float x[16];
            const int r = (sp & 1) * 32 + lane, cw = (sp >> 1) * 64 + q4 * 16;
            tc::tmem_ld16(tmem + tl + kTmW + cw, x);
            tc::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                x[i] = -x[i];
                ovf |= !(fabsf(x[i]) <= 65000.f);
            }
            *reinterpret_cast<uint4 *>(img + I::kNW + tile_chunk(r, cw / 8, kChunk)) = pack8_h(x);
            *reinterpret_cast<uint4 *>(img + I::kNW + tile_chunk(r, cw / 8 + 1, kChunk)) = pack8_h(x + 8);
            const int j = sp * 32 + lane;
            tc::tmem_ld16(tmem + tl + kTmUT + q4 * 16, x);
            tc::tmem_ld_wait();
            if (j < DV) {
#pragma unroll
                for (int i = 0; i < 16; ++i) ovf |= !(fabsf(x[i]) <= 65000.f);
                *reinterpret_cast<uint4 *>(img + I::kUT + tile_chunk(j, 2 * q4, DV)) = pack8_h(x);
                *reinterpret_cast<uint4 *>(img + I::kUT + tile_chunk(j, 2 * q4 + 1, DV)) = pack8_h(x + 8);
            }
        }
        tc::tc_fence_before();
        stage_done(ovf);
    }
    if (leader) drain_mma(&bars.fin, 0);
}

// ================================== chain role (cluster rank 0) =====================================
// The chain works on transposed tiles so that the state and U~ are the A operands of its MMAs,
// held in TMEM:
//   D1^T = S^T [-W ; Qg]^T        (columns 0-63: (U~ - U)^T, columns 64-127: (Qg S)^T)
//   D2^T = U~^T Kd                 (the state increment, transposed)
//   D1^T[:, 64:128] += U~^T P^T    (so that columns 64-127 become O^T)
// Warps 0-15 own the fp32 state: thread (warp w, lane l) holds value column j = 32 (w % 4) + l and key
// channels [32 (w / 4), 32 (w / 4) + 32) of S^T.  Lane 0 of warp 16 loads the chunk images.
template <int DV, typename TO>
__device__ __forceinline__ void chain_role(const ChunkCtx &cx, ChunkBars &bars, const RowMaps &maps,
                                           const __nv_bfloat16 *q,
                                           const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                                           const __nv_bfloat16 *log_alpha, const __nv_bfloat16 *beta,
                                           const float *init_state, TO *out, float *final_state) {
    using SM = ChainSmem<DV>;
    using I = Img<DV>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t *const sm = cx.sm;
    const uint32_t sbase = cx.sbase, tmem = cx.tmem;
    const int H = cx.H, h = cx.h, nchunks = cx.nchunks;
    volatile int *abort_flag = cx.abort_flag;

    if (warp >= kRoleWarps) {
        // ---- loader: producer region -> image slot c % 2, once the slot is free and the image published ----
        if (warp == kRoleWarps && lane == 0) {
            int last = -1;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                if (c >= 2) {
                    if (!tc::mbar_wait(&bars.slot_free[s], ((c >> 1) - 1) & 1, abort_flag)) break;
                    // chunk c - 2 has long been loaded: its producer may rewrite that region
                    const int pc = c - 2;
                    tc::mbar_arrive_cluster_relaxed(
                        tc::mapa(tc::smem_u32(&bars.consumed[(pc / kNP) & 1]), 1 + pc % kNP));
                }
                const int p = c % kNP, kq = c / kNP, reg = kq & 1;
                if (!tc::mbar_wait_cluster(&bars.pub[p][reg], (kq >> 1) & 1, abort_flag)) break;
                tc::fence_async_global();
                const uint8_t *src = cx.ws_pair + (size_t)(p * 2 + reg) * I::kStride;
                uint8_t *slot = sm + s * SM::kSlotBytes;
                uint64_t *fb = &bars.full[s];
                tc::mbar_arrive_expect_tx(fb, I::kBytes);
                tc::bulk_load(slot + SM::kA1, src + I::kNW, 8192, fb);
                tc::bulk_load(slot + SM::kA1 + 16384, src + I::kNW + 8192, 8192, fb);
                tc::bulk_load(slot + SM::kA1 + 8192, src + I::kQt, 8192, fb);
                tc::bulk_load(slot + SM::kA1 + 24576, src + I::kQt + 8192, 8192, fb);
                tc::bulk_load(slot + SM::kUT, src + I::kUT, kChunk * DV * 2, fb);
                tc::bulk_load(slot + SM::kKd, src + I::kKd, SM::kTailBytes, fb);
                last = c;
            }
            // no copy may still be in flight when the CTA leaves
            int never = 0;
            for (int c = (last >= 1 ? last - 1 : 0); c <= last; ++c)
                tc::mbar_wait(&bars.full[c & 1], (c >> 1) & 1, &never);
        }
        return;
    }

    const bool leader = tid == 0;
    const int sp = warp & 3, qd = warp >> 2;
    const int j = sp * 32 + lane;            // value column (TMEM lane)
    const bool jv = j < DV;
    const int c0 = qd * 32;                  // key channels [c0, c0 + 32)
    const uint32_t tl = tc::tmem_lane_base(warp);
    float *redPk = reinterpret_cast<float *>(sm + SM::kRedPk);
    float *redPq = reinterpret_cast<float *>(sm + SM::kRedPq);
    float *redKq = reinterpret_cast<float *>(sm + SM::kRedKq);

    float S[32];  // fp32 master state: S^T[j][c0 + i]
    const size_t state_base = ((size_t)cx.n * H + h) * kDK * DV + (size_t)c0 * DV + j;
#pragma unroll
    for (int i = 0; i < 32; ++i) S[i] = (init_state && jv) ? init_state[state_base + (size_t)i * DV] : 0.f;
    // S^T -> fp16 A operand in TMEM (lane j, channels c0..c0+31 in 16 columns); returns whether some
    // entry left the fp16 range
    auto write_state_operand = [&]() -> bool {
        bool big = false;
        uint32_t u[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            big |= !(fabsf(S[2 * i]) <= 65000.f) || !(fabsf(S[2 * i + 1]) <= 65000.f);
            u[i] = pack_h(S[2 * i], S[2 * i + 1]);
        }
        tc::tmem_st16(tmem + tl + kTmS + qd * 16, u);
        tc::tmem_st_wait();
        return big;
    };
    tc::tc_fence_before();
    bool force_exact = tc::named_sync_or(kBarRole, kRoleThreads, write_state_operand());

    // token-by-token fp32 evaluation of one chunk from the state in registers
    auto exact_chunk = [&](int64_t tok0, int L) -> bool {
        for (int r = 0; r < L; ++r) {
            const int64_t trow = (tok0 + r) * H + h;
            const __nv_bfloat16 *gr = log_alpha + trow * kDK + c0, *kr = k + trow * kDK + c0,
                                *qr = q + trow * kDK + c0;
            float pk = 0.f, pq = 0.f, kq = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float a = expf(__bfloat162float(gr[i])), kk = __bfloat162float(kr[i]),
                            qq = __bfloat162float(qr[i]);
                S[i] *= a;
                pk = fmaf(S[i], kk, pk);
                pq = fmaf(S[i], qq, pq);
                kq = fmaf(kk, qq, kq);
            }
            redPk[qd * 128 + j] = pk;
            redPq[qd * 128 + j] = pq;
            if (sp == 0 && lane == 0) redKq[qd] = kq;
            tc::named_sync(kBarRole, kRoleThreads);
            const float skq = (redKq[0] + redKq[1]) + (redKq[2] + redKq[3]);
            const float spk = (redPk[j] + redPk[128 + j]) + (redPk[256 + j] + redPk[384 + j]);
            const float spq = (redPq[j] + redPq[128 + j]) + (redPq[256 + j] + redPq[384 + j]);
            const float u = jv ? __bfloat162float(beta[trow]) * (__bfloat162float(v[trow * DV + j]) - spk) : 0.f;
            if (qd == 0 && jv) out[trow * DV + j] = from_f32<TO>(fmaf(u, skq, spq));
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] = fmaf(__bfloat162float(kr[i]), u, S[i]);
            tc::named_sync(kBarRole, kRoleThreads);
        }
        return write_state_operand();
    };

    // output of a tensor-path chunk: columns 64-127 of D1^T[b] hold O^T once [. ; P] U~ completed;
    // thread (j, qd) has tokens 16 qd + [0, 16) of value column j.  A full chunk is staged in
    // shared memory (a warp writes 32 consecutive values of one token: no bank conflicts) and written
    // by TMA tensor stores; a partial last chunk is stored directly.
    uint32_t ph_m3[2] = {0, 0};
    TO *const stage = reinterpret_cast<TO *>(sm + SM::kOut);
    auto store_output = [&](int cp, int bp) -> bool {
        if (leader) tc::bulk_wait_read_all();   // the previous chunk's stores have read the staging
        if (!role_wait(&bars.mma3[bp], ph_m3[bp], leader, kBarRole, kRoleThreads, abort_flag)) return false;
        ph_m3[bp] ^= 1u;
        float o[16];
        tc::tmem_ld16(tmem + tl + kTmD1 + bp * 128 + 64 + qd * 16, o);
        tc::tmem_ld_wait();
        const int64_t tok0 = cx.tok0(cp);
        const int L = cx.len(cp);
        if (L == kChunk) {
            if (jv) {
                TO *col = stage + (j >> 6) * (kChunk * 64) + (j & 63);
#pragma unroll
                for (int i = 0; i < 16; ++i) col[(qd * 16 + i) * 64] = from_f32<TO>(o[i]);
            }
            tc::fence_async_smem();
            tc::named_sync(kBarRole, kRoleThreads);
            if (leader) {
#pragma unroll
                for (int blk = 0; blk < DV / 64; ++blk)
                    tc::tma_store_3d(&maps.o, blk * 64, h, static_cast<int>(tok0), stage + blk * (kChunk * 64));
                tc::bulk_commit();
            }
        } else if (jv) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = qd * 16 + i;
                if (r < L) out[((tok0 + r) * H + h) * DV + j] = from_f32<TO>(o[i]);
            }
        }
        return true;
    };

    uint32_t ph1 = 0, ph2 = 0;
    bool prev_tensor = false;   // chunk c - 1 went through the tensor path: its output is pending
    for (int c = 0; c < nchunks; ++c) {
        const int s = c & 1, b = c & 1;
        const int64_t tok0 = cx.tok0(c);
        const int L = cx.len(c);
        const uint8_t *slot = sm + s * SM::kSlotBytes;
        const uint32_t sslot = sbase + s * SM::kSlotBytes;
        if (!role_wait(&bars.full[s], (c >> 1) & 1, leader, kBarRole, kRoleThreads, abort_flag)) break;
        const bool flagged = *reinterpret_cast<const volatile int *>(slot + SM::kFlag) != 0;
        if (!flagged && leader) {
            // ---- D1^T[b] = S^T [-W ; Qg]^T ----
            constexpr uint32_t id1 = tc::make_idesc(128, 128, tc::kF16, false, false);
#pragma unroll
            for (int kk = 0; kk < kDK / 16; ++kk)
                tc::mma_f16_ta(tmem + kTmD1 + b * 128, tmem + kTmS + kk * 8, desc_kmajor(sslot + SM::kA1, 128, kk),
                               id1, kk > 0);
            tc::mma_commit(&bars.mma1);
        }
        // the previous chunk's output, while D1^T[b] is computed; then its slot is free
        if (prev_tensor && !store_output(c - 1, b ^ 1)) break;
        if (c >= 1 && leader) tc::mbar_arrive(&bars.slot_free[s ^ 1]);
        prev_tensor = false;
        if (!flagged) {
            if (!role_wait(&bars.mma1, ph1, leader, kBarRole, kRoleThreads, abort_flag)) break;
            ph1 ^= 1u;
            // ---- U~^T = U^T + (-W S)^T (tokens 16 qd + [0, 16)) -> fp16 A operand in TMEM ----
            bool mybad = force_exact;
            {
                float x[16];
                tc::tmem_ld16(tmem + tl + kTmD1 + b * 128 + qd * 16, x);
                tc::tmem_ld_wait();
                uint32_t u[8];
                if (jv) {
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        float u8[8];
                        unpack8_h(*reinterpret_cast<const uint4 *>(slot + SM::kUT + tile_chunk(j, 2 * qd + h2, DV)),
                                  u8);
#pragma unroll
                        for (int i = 0; i < 8; ++i) x[8 * h2 + i] += u8[i];
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) mybad |= !(fabsf(x[i]) <= 65000.f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) u[i] = pack_h(x[2 * i], x[2 * i + 1]);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) u[i] = 0u;
                }
                tc::tmem_st8(tmem + tl + kTmUt + qd * 8, u);
                tc::tmem_st_wait();
            }
            tc::tc_fence_before();
            const bool bad = tc::named_sync_or(kBarRole, kRoleThreads, mybad);
            if (leader) {
                tc::tc_fence_after();
                // ---- D2^T = U~^T Kd;  D1^T[b][:, 64:128] += U~^T P^T ----
                constexpr uint32_t id2 = tc::make_idesc(128, 128, tc::kF16, false, true);
                constexpr uint32_t id3 = tc::make_idesc(128, kChunk, tc::kF16, false, false);
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk)
                    tc::mma_f16_ta(tmem + kTmD2, tmem + kTmUt + kk * 8, desc_mnmajor(sslot + SM::kKd, kChunk, kk),
                                   id2, kk > 0);
                tc::mma_commit(&bars.mma2);
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk)
                    tc::mma_f16_ta(tmem + kTmD1 + b * 128 + 64, tmem + kTmUt + kk * 8,
                                   desc_kmajor(sslot + SM::kP, kChunk, kk), id3, true);
                tc::mma_commit(&bars.mma3[b]);
            }
            if (!role_wait(&bars.mma2, ph2, leader, kBarRole, kRoleThreads, abort_flag)) break;
            ph2 ^= 1u;
            if (!bad) {
                // ---- S^T = S^T Diag(gamma) + D2^T ----
                const float4 *gam4 = reinterpret_cast<const float4 *>(slot + SM::kGam) + c0 / 4;
                {
                    float d[32];
                    tc::tmem_ld32(tmem + tl + kTmD2 + c0, d);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 gg = gam4[i4];
                        const int i = 4 * i4;
                        S[i] = fmaf(gg.x, S[i], d[i]);
                        S[i + 1] = fmaf(gg.y, S[i + 1], d[i + 1]);
                        S[i + 2] = fmaf(gg.z, S[i + 2], d[i + 2]);
                        S[i + 3] = fmaf(gg.w, S[i + 3], d[i + 3]);
                    }
                }
                const bool big = write_state_operand();
                tc::tc_fence_before();
                force_exact = tc::named_sync_or(kBarRole, kRoleThreads, big);
                prev_tensor = true;
                continue;
            }
            // this chunk is evaluated exactly: its pending [. ; P] U~ must still complete
            if (!role_wait(&bars.mma3[b], ph_m3[b], leader, kBarRole, kRoleThreads, abort_flag)) break;
            ph_m3[b] ^= 1u;
        }
        // exact path: the chunk's decays exceed the rebasing range, or an fp16 value overflowed
        const bool big = exact_chunk(tok0, L);
        tc::tc_fence_before();
        force_exact = tc::named_sync_or(kBarRole, kRoleThreads, big);
    }
    if (prev_tensor && nchunks > 0) store_output(nchunks - 1, (nchunks - 1) & 1);
    if (leader) tc::bulk_wait_all();   // every output store has completed before the CTA leaves
    if (final_state && *abort_flag == 0 && jv) {
#pragma unroll
        for (int i = 0; i < 32; ++i) final_state[state_base + (size_t)i * DV] = S[i];
    }
    if (leader) drain_mma(&bars.fin, 0);
}

// ====================================== kernel and launch ==========================================
template <int DV, typename TO>
__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_tc_kernel(const __grid_constant__ RowMaps maps, const __nv_bfloat16 *__restrict__ q,
                    const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
                    const __nv_bfloat16 *__restrict__ log_alpha, const __nv_bfloat16 *__restrict__ beta,
                    const float *init_state, const int32_t *__restrict__ cu_seqlens, int num_seqs, int T, int H,
                    TO *__restrict__ out, float *final_state, uint8_t *__restrict__ workspace) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ ChunkBars bars;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ int s_slot;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int rank = static_cast<int>(tc::cluster_ctarank());
    const int pair = blockIdx.x / kCL;
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

    if (tid == 0) {
        tc::mbar_init(&bars.full[0], 1);
        tc::mbar_init(&bars.full[1], 1);
        tc::mbar_init(&bars.slot_free[0], 1);
        tc::mbar_init(&bars.slot_free[1], 1);
        tc::mbar_init(&bars.mma1, 1);
        tc::mbar_init(&bars.mma2, 1);
        tc::mbar_init(&bars.mma3[0], 1);
        tc::mbar_init(&bars.mma3[1], 1);
        for (int p = 0; p < kNP; ++p) {
            tc::mbar_init(&bars.pub[p][0], 1);
            tc::mbar_init(&bars.pub[p][1], 1);
        }
        tc::mbar_init(&bars.m_ap, 1);
        tc::mbar_init(&bars.m_wu, 1);
        tc::mbar_init(&bars.consumed[0], 1);
        tc::mbar_init(&bars.consumed[1], 1);
        tc::mbar_init(&bars.staged, 1);
        tc::mbar_init(&bars.staging_free, 1);
        tc::mbar_init(&bars.raw_full, 1);
        tc::mbar_init(&bars.raw_free, 1);
        tc::mbar_init(&bars.fin, 1);
        tc::fence_mbar_init();
        abort_flag = 0;
    }
    const uint32_t ncols = rank == 0 ? kTmChainCols : kTmPrepCols;
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base_sh, ncols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync();  // every CTA's barriers are initialised before any remote arrive
    tc::tc_fence_after();

    ChunkCtx cx;
    cx.n = n;
    cx.h = h;
    cx.H = H;
    cx.t0 = t0;
    cx.t1 = t1;
    cx.nchunks = static_cast<int>((t1 - t0 + kChunk - 1) / kChunk);
    cx.sm = sm;
    cx.sbase = tc::smem_u32(sm);
    cx.tmem = tmem_base_sh;
    cx.ws_pair = workspace + (size_t)pair * kNP * 2 * Img<DV>::kStride;
    cx.abort_flag = &abort_flag;
    if (rank == 0)
        chain_role<DV, TO>(cx, bars, maps, q, k, v, log_alpha, beta, init_state, out, final_state);
    else
        prep_role<DV>(cx, bars, rank - 1, maps, beta);

    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync();  // no CTA leaves while a peer may still signal its barriers
    if (warp == 0) tc::tmem_dealloc(cx.tmem, ncols);
}

// Bytes of global workspace kda_chunk_fwd needs on the tensor-core path: two chunk
// image regions per (sequence, head) and prep CTA.
inline size_t chunk_tc_workspace_bytes(int64_t pairs, int DV) {
    return static_cast<size_t>(pairs) * kNP * 2 * (DV == 64 ? Img<64>::kStride : Img<128>::kStride);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// Map of a [tokens][H][d] tensor (bf16 or fp32) with boxes of 64 tokens x `box0` channels of one head.
inline bool encode_row_map(CUtensorMap *m, const void *base, int d, int H, int64_t tokens, int box0 = 0,
                           CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, int esize = 2) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(tokens)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esize, static_cast<cuuint64_t>(H) * d * esize};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box0 ? box0 : d), 1, kChunk};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DV, typename TO>
cudaError_t launch_chunk_tc_dv(const void *q, const void *k, const void *v, const void *la, const void *beta,
                               const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H,
                               void *out, float *final_state, void *workspace, cudaStream_t stream) {
    auto kern = kda_chunk_tc_kernel<DV, TO>;
    const int smem = chunk_smem_bytes<DV>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int N = cu ? num_seqs : B;
    RowMaps maps;
    memset(&maps, 0, sizeof(maps));
    const int64_t tokens = (int64_t)B * T;
    if (tokens > 0) {   // with no tokens no chunk is loaded and the maps stay unused
        if (!encode_row_map(&maps.g, la, kDK, H, tokens) || !encode_row_map(&maps.k, k, kDK, H, tokens) ||
            !encode_row_map(&maps.q, q, kDK, H, tokens) || !encode_row_map(&maps.v, v, DV, H, tokens) ||
            !encode_row_map(&maps.o, out, DV, H, tokens, 64,
                            sizeof(TO) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                            static_cast<int>(sizeof(TO))))
            return cudaErrorInvalidValue;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(N) * H * kCL);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, kern, maps, static_cast<const __nv_bfloat16 *>(q),
                              static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v),
                              static_cast<const __nv_bfloat16 *>(la), static_cast<const __nv_bfloat16 *>(beta),
                              init_state, cu, num_seqs, T, H, static_cast<TO *>(out), final_state,
                              static_cast<uint8_t *>(workspace));
}

template <typename TO>
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const void *la, const void *beta,
                            const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H, int DV,
                            void *out, float *final_state, void *workspace, cudaStream_t stream) {
    if (DV == 64)
        return launch_chunk_tc_dv<64, TO>(q, k, v, la, beta, init_state, cu, num_seqs, B, T, H, out, final_state,
                                          workspace, stream);
    return launch_chunk_tc_dv<128, TO>(q, k, v, la, beta, init_state, cu, num_seqs, B, T, H, out, final_state,
                                       workspace, stream);
}

}  // namespace kda
