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
// other quantity depends on the chunk's own inputs alone.  One grid, every CTA
// resident at once (cooperative launch), one CTA per SM:
//   * chain CTAs (one per (sequence, head) pair in flight; a chain runs its
//     pairs one after another) copy each chunk image from the chain's ring in a
//     global workspace (it stays in L2) into one of two shared-memory slots (image
//     t + 2 goes into chunk t's slot once chunk t's last MMA has completed), and
//     run, per chunk, one MMA group [-W ; Qg] S (rows 0-63 give U~ - U, rows
//     64-127 give Qg S), the U~ epilogue, the MMAs Kd^T U~ and [. ; P] U~ (adding
//     P U~ to rows 64-127) and the fp32 state update, while dedicated warps store
//     the output rows;
//   * producer CTAs (all other SMs, shared by all chains) prepare the chunks in
//     the order the chains need them: decays, rebased operands, A and P, the UT
//     transform, then W and U on the tensor cores.  The finished chunk image (-W,
//     U, Qg = Q exp(G), Kd = K exp(G_last - G), P, gamma = exp(G_last) and a
//     flag) is bulk-stored into its ring slot and announced through a flag in
//     global memory (after the store has completed and the async proxy is fenced,
//     a GPU-scope release store; the chain reads the flag with acquire loads and
//     fences the async proxy before its bulk copy of the image); the chain
//     announces in turn which slots it has copied out.
// Every producer serves every chain, so the preparation throughput per pair is
// (SMs - chains) / chains producer CTAs rather than a fixed cluster share.
// The chain CTA computes all d_v columns of S at once: a tcgen05.mma costs about
// the same for N = 32 and N = 128 value columns, so slicing d_v across CTAs would
// multiply the tensor-core time of the chain without shortening it.
//
// Precision (fp32 accumulation in TMEM, fp32 master state in registers, fp32
// decays and substitution, fp32 or bf16 output):
//   * A and P need the rebased factors below, whose range exceeds fp16: they are
//     one tf32 product (fp32 operands read with an 11-bit significand and the fp32
//     exponent range), [Kr ; Qr] Kn^T; the UT transform then runs in fp32.
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
//
// Input forms (template argument GK, see GateKind): one log-decay per key channel (KDA), one per
// head and token (Gated DeltaNet; none at all for DeltaNet), or KDA from the raw projections (q
// and k L2-normalised, log_alpha = logsigmoid(g), beta = sigmoid(b), all as they are loaded).
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

constexpr int kRoleWarps = 16;                        // warps 0-15 run the role
constexpr int kRoleThreads = kRoleWarps * 32;
constexpr int kThreads = kRoleThreads + 128;          // + four helper warps that move data
constexpr uint32_t kBarRole = 1, kBarOut = 2;          // named barriers: role warps, helper warps
constexpr uint32_t kBarUt = 3;                         // producer warps 0-7 inside the UT transform

// ---- chunk image (fp16 tiles in their shared-memory layouts) -----------------------------------
// The same bytes serve as the producer's staging area, the ring slot in the global workspace and the
// chain's shared-memory slot, so that one bulk copy moves a whole image.  A1 = [-W ; Qg] as two 16 KB
// k-blocks of 128 rows (rows 0-63 -W, rows 64-127 Qg: the B operand of S^T [-W ; Qg]^T), then U^T,
// Kd, tril(P), gamma = exp(G_last) and the exact-path flag.
template <int DV> struct Img {
    static constexpr int kA1 = 0;                          // [-W ; Qg] [128 x 128]
    static constexpr int kUT = kA1 + 2 * kChunk * kDK * 2; // U^T [DV x 64]
    static constexpr int kKd = kUT + kChunk * DV * 2;      // Kd  [64 x 128]
    static constexpr int kP = kKd + kChunk * kDK * 2;      // tril(P) [64 x 64]
    static constexpr int kGam = kP + kChunk * kChunk * 2;  // fp32 [128] exp(G_last)
    static constexpr int kFlag = kGam + kDK * 4;           // int: 1 = evaluate exactly
    static constexpr int kBytes = kFlag + 16;
    static constexpr int kStride = (kBytes + 1023) / 1024 * 1024;
    static_assert(kBytes % 16 == 0, "bulk copies move multiples of 16 bytes");
};
// Byte offsets of row r's 16-byte chunk j (8 channels) of -W and of Qg inside A1.
__device__ __forceinline__ uint32_t a1_nw(int r, int j) { return (j >> 3) * (2 * kChunk * 128) + tc::sw128(r, j & 7); }
__device__ __forceinline__ uint32_t a1_qg(int r, int j) { return a1_nw(r + kChunk, j); }

// ---- chain CTA shared memory ------------------------------------------------------------------
template <int DV> struct ChainSmem {
    using I = Img<DV>;
    // two image slots (Img layout); a slot is free again once the last MMA of its chunk completed
    static constexpr int kSlotBytes = I::kStride;
    static constexpr int kSlots = 2;
    // two output staging buffers (fp32 or bf16 [DV / 64 blocks][64 tokens][64 values]), so that a
    // chunk's TMA output store never holds up the reuse of an image slot
    static constexpr int kStageBytes = kChunk * DV * 4;
    static constexpr int kStage = kSlots * kSlotBytes;
    // exact path scratch (fp32): per-column partial sums of S^T k and S^T q per channel quarter, k . q
    static constexpr int kRedPk = kStage + 2 * kStageBytes;
    static constexpr int kRedPq = kRedPk + 4 * 128 * 4;
    static constexpr int kRedKq = kRedPq + 4 * 128 * 4;
    static constexpr int kBytes = kRedKq + 16;
};

// ---- prep CTA shared memory -------------------------------------------------------------------
template <int DV> struct PrepSmem {
    using I = Img<DV>;
    static constexpr int kTile = kChunk * kDK * 2;         // [64 x 128] 16-bit tile
    // fp32 (tf32) operands of the A/P product, K-major SW128 in 32-channel blocks of 128-byte rows:
    // A = [Kr ; Qr] (per block b: rows 0-63 K exp(G - Gref), rows 64-127 Q exp(G - Gref); 16 KB),
    // B = Kn = K exp(Gref - G) (per block: 64 rows, 8 KB)
    static constexpr int kKQBlk = 2 * kChunk * 128;
    static constexpr int kKnBlk = kChunk * 128;
    static constexpr int kKQ = 0;
    static constexpr int kKn = 4 * kKQBlk;
    static constexpr int kKgV = kKn + 4 * kKnBlk;          // [K exp(G) | V] [64 x 256], V zero past DV
    // [Tb | Tb]: the A operand of W (both row halves give the same rows, so all warps can read
    // them); the first Tb is also the B operand of U^T = V^T Tb^T
    static constexpr int kTbP = kKgV + kChunk * 2 * kDK * 2;
    static constexpr int kImg = kTbP + 2 * kChunk * kChunk * 2;  // staging image (Img layout)
    static constexpr int kG0 = kImg + I::kStride;                // fp32 [128] decay after token 0
    static constexpr int kGref = kG0 + kDK * 4;                  //            after token 31
    static constexpr int kGlast = kGref + kDK * 4;               //            after token 63
    static constexpr int kEref = kGlast + kDK * 4;               // exp(Gref)
    static constexpr int kElast = kEref + kDK * 4;               // exp(Glast - Gref)
    static constexpr int kBetaIn = kElast + kDK * 4;              // fp32 [2][64] beta of items kl, kl + 1
    static constexpr int kLenIn = kBetaIn + 2 * kChunk * 4;       // int [2] valid tokens (-1: no item)
    static constexpr int kBytes = kLenIn + 16;
    // The A/P operand area also holds, in turn: the raw bf16 inputs of the chunk (bulk-loaded
    // rows of log_alpha, k, q, v; read into registers before the operands are written) and the
    // fp32 scratch of the UT transform (once the A/P products complete).
    static constexpr int kRawG = 0, kRawK = kChunk * 256, kRawQ = 2 * kChunk * 256, kRawV = 3 * kChunk * 256;
    static constexpr int kRawBytes = kChunk * (3 * kDK * 2 + DV * 2);   // one TMA box per tensor
    static constexpr int kLd = 68;                               // row stride of A and T
    static constexpr int kA32 = 0;                               // A [64][68]
    static constexpr int kT32 = kA32 + kChunk * kLd * 4;         // T [64][68]
    static constexpr int kScr32 = kT32 + kChunk * kLd * 4;       // per-warp product tiles (warps 0-3)
    static constexpr int kScrFloats = 16 * 24;                   // [16][24] or [32][8]
    static_assert(kScr32 + 4 * kScrFloats * 4 <= kKgV && kRawV + kChunk * DV * 2 <= kKgV, "A/P operand area");
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
constexpr uint32_t kTmA = 0, kTmW = 256, kTmUT = 384, kTmPrepCols = 512;  // prep

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
// Finite fp32 -> nearest tf32 value (ties away from zero: add half a unit of the 10-bit significand,
// then clear the 13 low bits), still as an fp32 bit pattern
__device__ __forceinline__ float round_tf32(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xffffe000u);
}
__device__ __forceinline__ uint4 pack8_h(const float *f) {
    return make_uint4(pack_h(f[0], f[1]), pack_h(f[2], f[3]), pack_h(f[4], f[5]), pack_h(f[6], f[7]));
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
// Wait (bounded, ignoring the abort flag) for all tcgen05 operations this thread issued.
__device__ __forceinline__ void drain_mma(uint64_t *bar, uint32_t parity) {
    int never = 0;
    tc::mma_commit(bar);
    tc::mbar_wait(bar, parity, &never);
}

// Launch-wide schedule (computed on the host by launch_chunk_tc_dv) and its workspace tables.
// The grid has nchain chain CTAs and nprod producer CTAs, all resident at once (cooperative
// launch).  Chain k runs the (sequence, head) pairs k, k + nchain, ... one after another; its
// chunks, counted across those pairs, are numbered t = 0, 1, ...  Producer j prepares the items
// i = j, j + nprod, ..., item i being chunk t = i / nchain of chain k = i % nchain, and stores
// its image into slot t % ring of chain k's ring in the workspace.
struct ChunkSched {
    int npairs, nchain, nprod, ring, H, T;
    int C;                  // chunk length (1 <= C <= kChunk; a chunk of C < kChunk tokens fills the first C
                            // rows of the 64-row tiles, the rest are zero, as for the short last chunk)
    int dk;                 // key width of the inputs, 64 or kDK: with 64 the key channels 64-127 are zero
                            // (their state rows stay zero and never reach an output)
    const int32_t *cu;      // cu_seqlens, or null for [B, T] inputs
    const int32_t *order;   // sequences longest-first (packed inputs), or null for the identity
    int *ready;             // [nchain][ring]: 1 + number of the chunk whose image the slot holds
    int *consumed;          // [nchain]: chunks the chain has copied out of its ring
    uint8_t *rings;         // [nchain][ring] chunk images (Img layout, Img::kStride apart)
    tc::FlagWait fw;        // limit of the waits on the flags above, and the launch's abort word
    int skip_item;          // testing hook: the producer item whose image is never published (-1: none)
};

// One (sequence, head) pair.
struct PairInfo {
    int n, h, nchunks, C;
    int64_t t0, t1;
    // chunk c (C tokens, the last one shorter): first token and valid length (at most C <= kChunk)
    __device__ __forceinline__ int64_t tok0(int c) const { return t0 + (int64_t)c * C; }
    __device__ __forceinline__ int len(int c) const {
        const int64_t r = t1 - tok0(c);
        return static_cast<int>(r < C ? r : C);
    }
};
__device__ __forceinline__ PairInfo pair_info(const ChunkSched &s, int p) {
    PairInfo r;
    r.h = p % s.H;
    const int rank = p / s.H;
    if (s.cu) {
        r.n = s.order ? s.order[rank] : rank;
        r.t0 = s.cu[r.n];
        r.t1 = s.cu[r.n + 1];
    } else {
        r.n = rank;
        r.t0 = (int64_t)rank * s.T;
        r.t1 = r.t0 + s.T;
    }
    r.C = s.C;
    r.nchunks = static_cast<int>((r.t1 - r.t0 + s.C - 1) / s.C);
    return r;
}
// Chunk t of chain k: its pair and chunk index there; false if the chain has fewer chunks.
__device__ __forceinline__ bool chain_chunk(const ChunkSched &s, int k, int t, PairInfo &pi, int &c) {
    if (!s.cu) {   // equal lengths: direct
        pi = pair_info(s, k);
        if (pi.nchunks == 0) return false;
        const int q = t / pi.nchunks, p = k + q * s.nchain;
        if (p >= s.npairs) return false;
        pi = pair_info(s, p);
        c = t - q * pi.nchunks;
        return true;
    }
    for (int p = k; p < s.npairs; p += s.nchain) {
        pi = pair_info(s, p);
        if (t < pi.nchunks) {
            c = t;
            return true;
        }
        t -= pi.nchunks;
    }
    return false;
}
// Largest number of chunks any chain runs.
__device__ __forceinline__ int chain_tmax(const ChunkSched &s) {
    int tmax = 0;
    for (int k = 0; k < s.nchain; ++k) {
        int tot = 0;
        for (int p = k; p < s.npairs; p += s.nchain) tot += pair_info(s, p).nchunks;
        tmax = tot > tmax ? tot : tmax;
        if (!s.cu) break;   // equal lengths: chain 0 runs the most pairs
    }
    return tmax;
}

// Per-CTA bookkeeping shared by both roles.
struct ChunkCtx {
    uint32_t sbase, tmem;
    uint8_t *sm;
    volatile int *abort_flag;
};

// Mbarriers of one CTA (each role uses its own subset).
struct ChunkBars {
    // chain: image slot full, MMA completions
    uint64_t full[2], mma1, mma2, mma3[2];
    // chain: 1 + the chunk in which some state thread saw an fp16 overflow of U~ (ut) or of the state
    // operand (st); set before a plain barrier and compared with the chunk after it
    int ovf_ut, ovf_st;
    // chain: chunk evaluation mode handed to the output warps, TMEM accumulator read by them
    uint64_t outq[2], d1_free[2];
    int outmode[2];   // 0: no MMAs issued, 1: MMAs issued but evaluated exactly, 2: tensor output
    // chain: a state warp's own wait for MMA1 / MMA2 ran out (set before the barrier that follows
    // the wait, read after it, so that every state warp leaves at the same point)
    int fail1, fail2;
    // prep: MMA completions, staging image and raw input tiles
    uint64_t m_ap, m_wu, staged, staging_free, raw_full, raw_free;
    uint64_t fin;
};

// Tensor maps of the token tensors: [tokens][H][d] bf16, one box = 64 tokens x d channels of one
// head; and of the output [tokens][H][d_v] (fp32 or bf16), one box = 64 tokens x 64 values.
struct RowMaps {
    CUtensorMap g, k, q, v, o;
};

// ---- warp-level tf32 MMAs for the small products of the UT transform ----------------------------
// Fragment layouts of mma.sync m16n8k8 (tf32): with g = lane / 4 and t = lane % 4, A (16 x 8) holds
// (g, t), (g + 8, t), (g, t + 4), (g + 8, t + 4); B (8 x 8) holds (t, g), (t + 4, g); C (16 x 8) holds
// (g, 2t), (g, 2t + 1), (g + 8, 2t), (g + 8, 2t + 1).
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_16x8x8_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// acc (+)= A[16 x 8 KS] B[8 KS x 8], row-major fp32 operands in shared memory (leading dimensions la, lb)
template <int KS>
__device__ __forceinline__ void mma_tile_16x8(float (&acc)[4], const float *A, int la, const float *B, int lb, int g,
                                              int t) {
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        const float *a = A + 8 * ks, *b = B + 8 * ks * lb;
        const uint32_t af[4] = {to_tf32(a[g * la + t]), to_tf32(a[(g + 8) * la + t]), to_tf32(a[g * la + t + 4]),
                                to_tf32(a[(g + 8) * la + t + 4])};
        const uint32_t bf[2] = {to_tf32(b[t * lb + g]), to_tf32(b[(t + 4) * lb + g])};
        mma_16x8x8_tf32(acc, af, bf);
    }
}
// acc = A[16 x K] B[K x 16] as two 16 x 8 column tiles (K = 16)
template <int K>
__device__ __forceinline__ void mma_block_16x16(float (&acc)[2][4], const float *A, int la, const float *B, int lb,
                                                int g, int t) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        mma_tile_16x8<K / 8>(acc[nt], A, la, B + 8 * nt, lb, g, t);
    }
}

// ======================================== producer role ==========================================
// Producer j prepares its items (see ChunkSched) with warps 0-15.  Lane 0 of warp 16 stores each
// finished image into its ring slot once the chain has copied out the slot's previous image, and
// publishes it; lane 0 of warp 17 loads the raw input tiles of the next item.

// The producer's current item: chunk t of chain k, i.e. chunk c of pair pi.
struct ProdItem {
    int i, k, t, c;
    PairInfo pi;
};
// Advance `it` to the producer's next item (it.i + nprod, ...), skipping chunks past a chain's end;
// false once no chain has chunk t any more.
__device__ __forceinline__ bool next_item(const ChunkSched &s, int tmax, ProdItem &it) {
    for (int i = it.i + s.nprod;; i += s.nprod) {
        const int t = i / s.nchain, k = i - t * s.nchain;
        if (t >= tmax) return false;
        if (chain_chunk(s, k, t, it.pi, it.c)) {
            it.i = i;
            it.k = k;
            it.t = t;
            return true;
        }
    }
}
__device__ __forceinline__ bool first_item(const ChunkSched &s, int tmax, int j, ProdItem &it) {
    it.i = j - s.nprod;
    return next_item(s, tmax, it);
}

template <int DV, int GK>
__device__ __forceinline__ void prep_role(const ChunkCtx &cx, ChunkBars &bars, const ChunkSched &sched, int j,
                                          int tmax, const RowMaps &maps, const __nv_bfloat16 *log_g,
                                          const __nv_bfloat16 *beta) {
    using SM = PrepSmem<DV>;
    using I = Img<DV>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t *const sm = cx.sm;
    const uint32_t sbase = cx.sbase, tmem = cx.tmem;
    const int H = sched.H;
    volatile int *abort_flag = cx.abort_flag;
    if (warp == kRoleWarps) {
        if (lane == 0) {
            // ---- publisher: staged image -> its ring slot (one bulk store), then announce it ----
            ProdItem it;
            bool have = first_item(sched, tmax, j, it);
            for (int kl = 0; have; ++kl, have = next_item(sched, tmax, it)) {
                const int slot = it.t % sched.ring;
                uint8_t *gimg = sched.rings + ((size_t)it.k * sched.ring + slot) * I::kStride;
                // the chain has copied out the slot's previous image (chunk t - ring)
                if (!tc::flag_wait_ge(sched.consumed + it.k, it.t - sched.ring + 1, abort_flag, sched.fw)) break;
                if (!tc::mbar_wait(&bars.staged, kl & 1, abort_flag)) break;
                if (it.i == sched.skip_item) {   // testing hook: this image is never published
                    tc::mbar_arrive(&bars.staging_free);
                    continue;
                }
                tc::fence_async_global();
                tc::bulk_store_nc(gimg, sm + SM::kImg, I::kBytes);
                tc::bulk_commit();
                tc::bulk_wait_read_all();
                tc::mbar_arrive(&bars.staging_free);
                tc::bulk_wait_all();
                tc::fence_async_global();
                tc::st_release_gpu(sched.ready + it.k * sched.ring + slot, it.t + 1);
            }
        }
        return;
    }
    if (warp >= kRoleWarps + 2) return;   // warps 18, 19 serve the chain CTA only
    if (warp == kRoleWarps + 1) {
        // ---- item loader: for each item, lane 0 issues the 64-token TMA tiles of the gate, k, q,
        //      v (rows past the tensor end read as zero, rows past the sequence end are masked by the
        //      readers) into the A/P operand area once the previous item's UT scratch is dead; the
        //      warp then stores the item's beta (and, for a per-head gate, the 64 log-decays in place
        //      of the gate tile) and length into shared memory.  raw_full completes
        //      with both arrivals and the tile bytes.  After the last item a length of -1 (no tiles)
        //      tells the compute warps to stop ----
        float *sBetaIn = reinterpret_cast<float *>(sm + SM::kBetaIn);
        int *sLenIn = reinterpret_cast<int *>(sm + SM::kLenIn);
        int last = -1;   // last raw_full phase this warp arrived on
        ProdItem it;
        bool have = first_item(sched, tmax, j, it);
        for (int kl = 0;; ++kl) {
            bool ok = true;
            if (lane == 0 && kl >= 1) ok = tc::mbar_wait(&bars.raw_free, (kl - 1) & 1, abort_flag);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const int64_t tok0 = have ? it.pi.tok0(it.c) : 0;
            const int L = have ? it.pi.len(it.c) : -1, h = it.pi.h;
            if (lane == 0) {
                // a per-head gate comes as 64 scalars (below) instead of a log_alpha tile
                const uint32_t kTileBytes = (GK != kGateHead ? 3u : 2u) * kChunk * sched.dk * 2 + kChunk * DV * 2;
                tc::mbar_arrive_expect_tx(&bars.raw_full, have ? kTileBytes : 0);
                if (have) {
                    const int t = static_cast<int>(tok0);
                    if constexpr (GK != kGateHead) tc::tma_load_3d(sm + SM::kRawG, &maps.g, 0, h, t, &bars.raw_full);
                    tc::tma_load_3d(sm + SM::kRawK, &maps.k, 0, h, t, &bars.raw_full);
                    tc::tma_load_3d(sm + SM::kRawQ, &maps.q, 0, h, t, &bars.raw_full);
                    tc::tma_load_3d(sm + SM::kRawV, &maps.v, 0, h, t, &bars.raw_full);
                }
            }
            float *bdst = sBetaIn + (kl & 1) * kChunk;
            bdst[lane] = (lane < L) ? beta_of<GK>(beta, (size_t)(tok0 + lane) * H + h) : 0.f;
            bdst[32 + lane] = (32 + lane < L) ? beta_of<GK>(beta, (size_t)(tok0 + 32 + lane) * H + h) : 0.f;
            if constexpr (GK == kGateHead) {   // fp32 log-decays of the 64 tokens, in place of the tile
                float *gdst = reinterpret_cast<float *>(sm + SM::kRawG);
                gdst[lane] = (lane < L) ? gate_log<GK>(log_g, (size_t)(tok0 + lane) * H + h, kDK, 0) : 0.f;
                gdst[32 + lane] =
                    (32 + lane < L) ? gate_log<GK>(log_g, (size_t)(tok0 + 32 + lane) * H + h, kDK, 0) : 0.f;
            }
            if (lane == 0) sLenIn[kl & 1] = L;
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars.raw_full);
            last = kl;
            if (!have) break;
            have = next_item(sched, tmax, it);
        }
        // no copy may still be in flight when the CTA leaves (phases complete in order)
        if (lane == 0 && last >= 0) {
            int never = 0;
            tc::mbar_wait(&bars.raw_full, last & 1, &never);
        }
        return;
    }

    // ---- compute warps 0-15 ----
    const int dkin = sched.dk;   // key channels present in the input rows (the rest read as zero)
    const int tp = tid;
    const bool leader = tp == 0;
    const int cg = tp & 15, tg = tp >> 4;   // channels [8cg, 8cg+8), tokens 2tg, 2tg + 1
    const int sp = warp & 3, q4 = warp >> 2;
    const uint32_t tl = tc::tmem_lane_base(warp);
    const int *sLenIn = reinterpret_cast<const int *>(sm + SM::kLenIn);
    float *sG0 = reinterpret_cast<float *>(sm + SM::kG0);
    float *sGref = reinterpret_cast<float *>(sm + SM::kGref);
    float *sGlast = reinterpret_cast<float *>(sm + SM::kGlast);
    float *sTot = reinterpret_cast<float *>(sm + SM::kTot);
    float *sPre = reinterpret_cast<float *>(sm + SM::kPre);
    constexpr int ld = SM::kLd;
    float *sA = reinterpret_cast<float *>(sm + SM::kA32);
    float *sT = reinterpret_cast<float *>(sm + SM::kT32);
    float *sS = reinterpret_cast<float *>(sm + SM::kScr32);

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
    for (int kl = 0;; ++kl) {
        // the raw inputs, beta and length of the item are in shared memory
        if (!role_wait(&bars.raw_full, kl & 1, leader, kBarRole, kRoleThreads, abort_flag)) break;
        const int L = sLenIn[kl & 1];
        if (L < 0) break;   // no more items
        const float *sBeta = reinterpret_cast<const float *>(sm + SM::kBetaIn) + (kl & 1) * kChunk;
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
                if constexpr (GK != kGateHead) {
                    const uint4 raw = (r < L && cg * 8 < dkin)
                                          ? *reinterpret_cast<const uint4 *>(sm + SM::kRawG + r * dkin * 2 + cg * 16)
                                            : make_uint4(0, 0, 0, 0);
                    unpack8(raw, g8);
                    if constexpr (GK == kRawInputs) {   // the gate's pre-activation: log_alpha = logsigmoid
#pragma unroll
                        for (int i = 0; i < 8; ++i) g8[i] = r < L ? log_sigmoid_fast(g8[i]) : 0.f;
                    }
                } else {   // one decay for every channel
                    const float gs = r < L ? reinterpret_cast<const float *>(sm + SM::kRawG)[r] : 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) g8[i] = gs;
                }
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
            reinterpret_cast<float *>(sm + SM::kEref)[tp] = fast_exp(gref);
            reinterpret_cast<float *>(sm + SM::kElast)[tp] = fast_exp(run - gref);
            bad = !((sG0[tp] - gref <= kRangeLimit) && (gref - run <= kRangeLimit));
        }
        if (tc::named_sync_or(kBarRole, kRoleThreads, bad)) {
            // decays too fast for the rebased products: the chain evaluates this chunk exactly
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
            const bool kin = in && cg * 8 < dkin;
            rk[rr] = kin ? *reinterpret_cast<const uint4 *>(sm + SM::kRawK + r * dkin * 2 + cg * 16) : make_uint4(0, 0, 0, 0);
            rq[rr] = kin ? *reinterpret_cast<const uint4 *>(sm + SM::kRawQ + r * dkin * 2 + cg * 16) : make_uint4(0, 0, 0, 0);
            rv[rr] = (in && cg * 8 < DV) ? *reinterpret_cast<const uint4 *>(sm + SM::kRawV + r * DV * 2 + cg * 16)
                                         : make_uint4(0, 0, 0, 0);
        }
        tc::named_sync(kBarRole, kRoleThreads);   // the operands below overwrite the raw rows
        {
            // fp32 operand rows: channels 8 cg .. 8 cg + 7 are 16-byte chunks 2 (cg % 4) and 2 (cg % 4) + 1
            // of 32-channel block cg / 4; lanes of odd blocks store the second chunk first, so that
            // each group of eight lanes covers all eight chunk positions of a row (no bank conflicts)
            const int c16 = 2 * (cg & 3);
            const bool swap = (cg >> 2) & 1;
            const uint32_t okq = SM::kKQ + (cg >> 2) * SM::kKQBlk, okn = SM::kKn + (cg >> 2) * SM::kKnBlk;
            // values are rounded to tf32 here (to nearest): the tensor cores would otherwise drop the
            // low mantissa bits, a bias that adds up coherently over the 128 channels of a product
            auto st_f32x8 = [&](uint32_t base, int row, const float *f) {
                float t[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) t[i] = round_tf32(f[i]);
                const float4 lo = make_float4(t[0], t[1], t[2], t[3]), hi = make_float4(t[4], t[5], t[6], t[7]);
                const uint32_t olo = base + tc::sw128(row, c16), ohi = base + tc::sw128(row, c16 + 1);
                *reinterpret_cast<float4 *>(sm + (swap ? ohi : olo)) = swap ? hi : lo;
                *reinterpret_cast<float4 *>(sm + (swap ? olo : ohi)) = swap ? lo : hi;
            };
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = tg * 2 + rr;
                float kf[8], qf[8];
                unpack8(rk[rr], kf);
                unpack8(rq[rr], qf);
                if constexpr (GK == kRawInputs) {
                    // raw q and k rows: L2-normalise over the 128 channels, which the 16 lanes of this
                    // half-warp hold 8 each
                    float sk = 0.f, sq = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        sk = fmaf(kf[i], kf[i], sk);
                        sq = fmaf(qf[i], qf[i], sq);
                    }
#pragma unroll
                    for (int o = 1; o < 16; o <<= 1) {
                        sk += __shfl_xor_sync(0xffffffffu, sk, o);
                        sq += __shfl_xor_sync(0xffffffffu, sq, o);
                    }
                    const float nk = rsqrtf(sk + kNormEps), nq = rsqrtf(sq + kNormEps);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        kf[i] *= nk;
                        qf[i] *= nq;
                    }
                }
                // per-channel constants, re-read from shared memory for each token (fewer live registers)
                float gref[8], eref[8], elast[8];
                const float *sEref = reinterpret_cast<const float *>(sm + SM::kEref) + cg * 8;
                const float *sElast = reinterpret_cast<const float *>(sm + SM::kElast) + cg * 8;
#pragma unroll
                for (int i4 = 0; i4 < 8; i4 += 4) {
                    *reinterpret_cast<float4 *>(gref + i4) = *reinterpret_cast<const float4 *>(sGref + cg * 8 + i4);
                    *reinterpret_cast<float4 *>(eref + i4) = *reinterpret_cast<const float4 *>(sEref + i4);
                    *reinterpret_cast<float4 *>(elast + i4) = *reinterpret_cast<const float4 *>(sElast + i4);
                }
                float kr[8], qr[8], kn[8], kd[8], kg[8], qg[8], vf[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float dg = G[rr][i] - gref[i];
                    const float e1 = fast_exp(dg), e2 = fast_exp(-dg);
                    kr[i] = kf[i] * e1;
                    qr[i] = qf[i] * e1;
                    kn[i] = kf[i] * e2;
                    kd[i] = kn[i] * elast[i];
                    kg[i] = kr[i] * eref[i];
                    qg[i] = qr[i] * eref[i];
                }
                const uint32_t o128 = tile_chunk(r, cg, kChunk);   // [64 x 128] tiles
                *reinterpret_cast<uint4 *>(sm + SM::kKgV + o128) = pack8_h(kg);
                *reinterpret_cast<uint4 *>(img + I::kA1 + a1_qg(r, cg)) = pack8_h(qg);
                unpack8(rv[rr], vf);   // zero past DV
#pragma unroll
                for (int i = 0; i < 8; ++i) ovf |= !(fabsf(vf[i]) <= 65000.f);
                *reinterpret_cast<uint4 *>(sm + SM::kKgV + tile_chunk(r, 16 + cg, kChunk)) = pack8_h(vf);
                st_f32x8(okq, r, kr);
                st_f32x8(okq, 64 + r, qr);
                st_f32x8(okn, r, kn);
                *reinterpret_cast<uint4 *>(img + I::kKd + o128) = pack8_h(kd);
            }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        tc::named_sync(kBarRole, kRoleThreads);

        // ---- A/P product (tf32): D = [Kr ; Qr] Kn^T: rows 0-63 A_raw, rows 64-127 P ----
        if (leader) {
            tc::tc_fence_after();
            constexpr uint32_t id = tc::make_idesc(128, 64, tc::kTF32, false, false);
#pragma unroll
            for (int kk = 0; kk < kDK / 8; ++kk) {
                const uint64_t a = tc::make_sdesc(sbase + SM::kKQ + (kk >> 2) * SM::kKQBlk + (kk & 3) * 32, 16, 1024,
                                                  tc::kSwz128);
                const uint64_t bd = tc::make_sdesc(sbase + SM::kKn + (kk >> 2) * SM::kKnBlk + (kk & 3) * 32, 16, 1024,
                                                   tc::kSwz128);
                tc::mma_tf32(tmem + kTmA, a, bd, id, kk > 0);
            }
            tc::mma_commit(&bars.m_ap);
        }
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
                tc::tmem_ld_wait();
                const int r = m - 64;
#pragma unroll
                for (int i = 0; i < 16; ++i) x16[i] = (cb + i <= r) ? x16[i] : 0.f;
                *reinterpret_cast<uint4 *>(img + I::kP + tile_chunk(r, cb / 8, kChunk)) = pack8_h(x16);
                *reinterpret_cast<uint4 *>(img + I::kP + tile_chunk(r, cb / 8 + 1, kChunk)) = pack8_h(x16 + 8);
            }
        }
        tc::tc_fence_before();
        tc::named_sync(kBarRole, kRoleThreads);

        // ---- UT transform T = (I + A)^{-1} (row-major in sT; blocks above the diagonal never written) ----
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
                sT[(16 * bb + pp + 8 * kq) * ld + 16 * bb + cc] = x[kq];
                // the upper blocks (0, 1) and (2, 3) are zero: the block products below read them
                if ((bb & 1) == 0) sT[(16 * bb + pp + 8 * kq) * ld + 16 * bb + 16 + cc] = 0.f;
            }
        }
        tc::named_sync(kBarRole, kRoleThreads);
        // (b) the blocks below the diagonal, as two levels of the 2x2 block inverse
        //     [[Ta, 0], [Lba, Tb']]^{-1} = [[Ta, 0], [-Tb' Lba Ta, Tb']]: level 1 (16-row blocks) gives
        //     T10 and T32, level 2 (32-row blocks) the lower-left 32x32 block.  The products run on
        //     warp-level tensor-core MMAs (m16n8k8, tf32 operands rounded to nearest, fp32
        //     accumulation); each product's result goes through the scratch tile to become the
        //     next product's operand.
        {
            float *sXs = sS;   // level 1: [2][16][kXld];  level 2: [32][kYld]
            constexpr int kXld = 20, kYld = 36;
            const int g = lane >> 2, t4 = lane & 3;
            // level 1: warp w < 2 forms T_ij for (i, j) = (2w + 1, 2w)
            if (warp < 2) {
                const int i = 2 * warp + 1, j = 2 * warp;
                float *X = sXs + warp * 16 * kXld;
                float acc[2][4];
                // X = A_ij T_jj
                mma_block_16x16<16>(acc, sA + 16 * i * ld + 16 * j, ld, sT + 16 * j * ld + 16 * j, ld, g, t4);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    X[g * kXld + 8 * nt + 2 * t4] = acc[nt][0];
                    X[g * kXld + 8 * nt + 2 * t4 + 1] = acc[nt][1];
                    X[(g + 8) * kXld + 8 * nt + 2 * t4] = acc[nt][2];
                    X[(g + 8) * kXld + 8 * nt + 2 * t4 + 1] = acc[nt][3];
                }
                __syncwarp();
                // T_ij = -T_ii X
                mma_block_16x16<16>(acc, sT + 16 * i * ld + 16 * i, ld, X, kXld, g, t4);
                float *Tij = sT + 16 * i * ld + 16 * j;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    *reinterpret_cast<float2 *>(Tij + g * ld + 8 * nt + 2 * t4) = make_float2(-acc[nt][0], -acc[nt][1]);
                    *reinterpret_cast<float2 *>(Tij + (g + 8) * ld + 8 * nt + 2 * t4) =
                        make_float2(-acc[nt][2], -acc[nt][3]);
                }
            }
            tc::named_sync(kBarRole, kRoleThreads);
            // level 2: warp w < 8 forms the 16 x 8 tile (mt, nt) = (w / 4, w % 4) of Y = Lba Ta, then of
            // Tba = -Tb' Y (Tb' is block lower triangular: rows 0-15 of it need only k < 16)
            if (warp < 8) {
                const int mt = warp >> 2, nt = warp & 3;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                mma_tile_16x8<4>(acc, sA + (32 + 16 * mt) * ld, ld, sT + 8 * nt, ld, g, t4);
                float *Y = sXs;
                *reinterpret_cast<float2 *>(Y + (16 * mt + g) * kYld + 8 * nt + 2 * t4) = make_float2(acc[0], acc[1]);
                *reinterpret_cast<float2 *>(Y + (16 * mt + g + 8) * kYld + 8 * nt + 2 * t4) =
                    make_float2(acc[2], acc[3]);
                tc::named_sync(kBarUt, 256);
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[e] = 0.f;
                if (mt == 0)
                    mma_tile_16x8<2>(acc, sT + 32 * ld + 32, ld, Y + 8 * nt, kYld, g, t4);
                else
                    mma_tile_16x8<4>(acc, sT + 48 * ld + 32, ld, Y + 8 * nt, kYld, g, t4);
                float *Tba = sT + (32 + 16 * mt) * ld + 8 * nt;
                *reinterpret_cast<float2 *>(Tba + g * ld + 2 * t4) = make_float2(-acc[0], -acc[1]);
                *reinterpret_cast<float2 *>(Tba + (g + 8) * ld + 2 * t4) = make_float2(-acc[2], -acc[3]);
            }
            tc::named_sync(kBarRole, kRoleThreads);
        }
        // T diag(beta) -> fp16 A operand [64 x 64], one chunk of 8 per thread; the strictly upper
        // blocks of T are never written, so the mask s <= r is applied here
        {
            const int r = tp >> 3, j = tp & 7;
            const float4 t0 = *reinterpret_cast<const float4 *>(sT + r * ld + 8 * j);
            const float4 t1 = *reinterpret_cast<const float4 *>(sT + r * ld + 8 * j + 4);
            const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = (j * 8 + i <= r) ? tv[i] * sBeta[j * 8 + i] : 0.f;
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
            *reinterpret_cast<uint4 *>(img + I::kA1 + a1_nw(r, cw / 8)) = pack8_h(x);
            *reinterpret_cast<uint4 *>(img + I::kA1 + a1_nw(r, cw / 8 + 1)) = pack8_h(x + 8);
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

// ========================================== chain role ===========================================
// The chain works on transposed tiles so that the state and U~ are the A operands of its MMAs,
// held in TMEM:
//   D1^T = S^T [-W ; Qg]^T        (columns 0-63: (U~ - U)^T, columns 64-127: (Qg S)^T)
//   D2^T = U~^T Kd                 (the state increment, transposed)
//   D1^T[:, 64:128] += U~^T P^T    (so that columns 64-127 become O^T)
// Warps 0-15 own the fp32 state: thread (warp w, lane l) holds value column j = 32 (w % 4) + l and key
// channels [32 (w / 4), 32 (w / 4) + 32) of S^T.  Warps 16-19 store the outputs; lane 1 of warp 16
// also copies the chunk images out of the chain's ring.  Chain kc runs the pairs kc, kc + nchain, ...;
// its chunks are numbered t across them (image slots, barrier phases and ring slots follow t).
template <int DV, typename TO, int GK>
__device__ __forceinline__ void chain_role(const ChunkCtx &cx, ChunkBars &bars, const ChunkSched &sched, int kc,
                                           const RowMaps &maps, const __nv_bfloat16 *q,
                                           const __nv_bfloat16 *k, const __nv_bfloat16 *v,
                                           const __nv_bfloat16 *log_alpha, const __nv_bfloat16 *beta,
                                           const float *init_state, TO *out, float *final_state) {
    using SM = ChainSmem<DV>;
    using I = Img<DV>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t *const sm = cx.sm;
    const uint32_t sbase = cx.sbase, tmem = cx.tmem;
    const int H = sched.H;
    volatile int *abort_flag = cx.abort_flag;
    int ttot = 0;   // chunks of this chain
    for (int p = kc; p < sched.npairs; p += sched.nchain) ttot += pair_info(sched, p).nchunks;

    if (warp >= kRoleWarps) {
        // ---- output and image warps 16-19: warp 16 + w reads TMEM lanes 32 w .. 32 w + 31, i.e. value
        //      columns j = 32 w + lane of O^T (columns 64-127 of D1^T[b]) once [. ; P] U~ completed, and
        //      stages them in their own double buffer for TMA tensor stores; lane 1 of warp 16 copies the
        //      chunk images from the chain's ring in global memory into the two slots: image t + 2 goes
        //      into chunk t's slot as soon as chunk t's last MMA has completed ----
        const int jo = (warp & 3) * 32 + lane;
        const bool jov = jo < DV;
        const bool lead = warp == kRoleWarps && lane == 0;
        // the image copies are issued by another lane than the output stores: the image lane's fence and
        // flag waits then do not wait for the output stores still in flight
        const bool lead_ld = warp == kRoleWarps && lane == 1;
        const uint32_t tlo = tc::tmem_lane_base(warp);
        constexpr uint32_t kOutThreads = kThreads - kRoleThreads;
        // chunk whose image copy was issued last into each slot (-1: none); copies into one slot are
        // sequential (each waits for the MMAs that read the previous one), so these are the only copies
        // that may be in flight when the CTA leaves
        int pend[SM::kSlots];
#pragma unroll
        for (int i = 0; i < SM::kSlots; ++i) pend[i] = -1;
        auto ready_flag = [&](int t) { return sched.ready + kc * sched.ring + t % sched.ring; };
        auto copy_image = [&](int t) {   // lane 1 of warp 16, once image t's ready flag has been seen
            tc::fence_async_global();
            const uint8_t *src = sched.rings + ((size_t)kc * sched.ring + t % sched.ring) * I::kStride;
            uint64_t *fb = &bars.full[t % SM::kSlots];
            tc::mbar_arrive_expect_tx(fb, I::kBytes);
            tc::bulk_load(sm + (t % SM::kSlots) * SM::kSlotBytes, src, I::kBytes, fb);   // one copy per image
            pend[t % SM::kSlots] = t;
        };
        if (lead_ld)
            for (int t = 0; t < SM::kSlots && t < ttot; ++t) {
                if (*abort_flag || !tc::flag_wait_ge(ready_flag(t), t + 1, abort_flag, sched.fw)) break;
                copy_image(t);
            }
        // a wait by lane 0 of warp 16, whose outcome all four warps share (they leave together)
        auto out_wait = [&](uint64_t *bar, uint32_t parity) -> bool {
            bool ok = true;
            if (lead) ok = tc::mbar_wait(bar, parity, abort_flag);
            const bool failed = tc::named_sync_or(kBarOut, kOutThreads, !ok);
            tc::tc_fence_after();
            return !failed;
        };
        uint32_t ph_q[2] = {0, 0}, ph3[2] = {0, 0};
        int t = 0;
        bool stop = false;
        for (int pr = kc; pr < sched.npairs && !stop; pr += sched.nchain) {
            const PairInfo pi = pair_info(sched, pr);
            const int h = pi.h;
            for (int c = 0; c < pi.nchunks; ++c, ++t) {
                const int b = t & 1;
                TO *stage = reinterpret_cast<TO *>(sm + SM::kStage + b * SM::kStageBytes);
                // the ready flag of image t + 2, read now (an acquire load) and used once chunk t's slot is
                // free, so that its latency overlaps the waits below
                const bool next = lead_ld && t + SM::kSlots < ttot;
                const int seen = next ? tc::ld_acquire_gpu(ready_flag(t + SM::kSlots)) : 0;
                // staging buffer b was last read by the TMA store of chunk t - 2 (at most one newer store,
                // chunk t - 1's, may still be reading its buffer); the barrier below publishes this
                if (lead) tc::bulk_wait_read_1();
                // the state warps have chosen how chunk t is evaluated (outmode) ...
                if (!out_wait(&bars.outq[b], ph_q[b])) {
                    stop = true;
                    break;
                }
                ph_q[b] ^= 1u;
                const int mode = *reinterpret_cast<volatile int *>(&bars.outmode[b]);
                // ... and, when its MMAs were issued, they have completed
                if (mode >= 1) {
                    if (!out_wait(&bars.mma3[b], ph3[b])) {
                        stop = true;
                        break;
                    }
                    ph3[b] ^= 1u;
                }
                // every read of chunk t's slot is over (the state warps read it before they issue the
                // chunk's last MMAs, or before they signal an exactly evaluated chunk): image t + 2 goes
                // there.  A failed flag wait sets the abort flag, which the next barrier wait turns into a stop.
                if (next && !*abort_flag &&
                    (seen >= t + SM::kSlots + 1 ||
                     tc::flag_wait_ge(ready_flag(t + SM::kSlots), t + SM::kSlots + 1, abort_flag, sched.fw)))
                    copy_image(t + SM::kSlots);
                if (mode == 2) {
                    const int64_t tok0 = pi.tok0(c);
                    const int L = pi.len(c);
                    const bool full = L == kChunk;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {   // tokens 32 half + [0, 32)
                        float o[32];
                        tc::tmem_ld32(tmem + tlo + kTmD1 + b * 128 + 64 + 32 * half, o);
                        tc::tmem_ld_wait();
                        if (half == 1) {
                            // D1^T[b] may be overwritten by the MMAs of chunk t + 2
                            tc::tc_fence_before();
                            __syncwarp();
                            if (lane == 0) tc::mbar_arrive(&bars.d1_free[b]);
                        }
                        if (!jov) continue;
                        if (full) {
                            TO *col = stage + (jo >> 6) * (kChunk * 64) + (jo & 63) + 32 * half * 64;
#pragma unroll
                            for (int i = 0; i < 32; ++i) col[i * 64] = from_f32<TO>(o[i]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (32 * half + i < L)
                                    out[((tok0 + 32 * half + i) * H + h) * DV + jo] = from_f32<TO>(o[i]);
                        }
                    }
                    if (full) {
                        tc::fence_async_smem();
                        tc::named_sync(kBarOut, kOutThreads);
                        if (lead) {
#pragma unroll
                            for (int blk = 0; blk < DV / 64; ++blk)
                                tc::tma_store_3d(&maps.o, blk * 64, h, static_cast<int>(tok0),
                                                 stage + blk * (kChunk * 64));
                        }
                    }
                } else {
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&bars.d1_free[b]);
                }
                // one bulk group per chunk (empty when the chunk had no TMA store), so that wait_group.read 1
                // at the top always names chunk t - 1's group
                if (lead) tc::bulk_commit();
            }
        }
        if (lead) tc::bulk_wait_all();   // every output store has completed before the CTA leaves
        if (lead_ld) {
            int never = 0;
#pragma unroll
            for (int i = 0; i < SM::kSlots; ++i)
                if (pend[i] >= 0) tc::mbar_wait(&bars.full[i], (pend[i] / SM::kSlots) & 1, &never);
        }
        return;
    }

    const bool leader = tid == 0;
    const int sp = warp & 3, qd = warp >> 2;
    const int j = sp * 32 + lane;            // value column (TMEM lane)
    const bool jv = j < DV;
    const int c0 = qd * 32;                  // key channels [c0, c0 + 32)
    const int dkin = sched.dk;               // key channels present in the inputs
    const bool kin = c0 < dkin;              // this thread's channels are (not padding)
    const uint32_t tl = tc::tmem_lane_base(warp);
    float *redPk = reinterpret_cast<float *>(sm + SM::kRedPk);
    float *redPq = reinterpret_cast<float *>(sm + SM::kRedPq);
    float *redKq = reinterpret_cast<float *>(sm + SM::kRedKq);

    float S[32];  // fp32 master state: S^T[j][c0 + i] of the current pair
    int h = 0;    // the current pair's head
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
    // token-by-token fp32 evaluation of one chunk from the state in registers
    auto exact_chunk = [&](int64_t tok0, int L) -> bool {
        for (int r = 0; r < L; ++r) {
            const int64_t trow = (tok0 + r) * H + h;
            // a per-head gate: the same log-decay for every channel (none when log_g is null)
            constexpr int gstride = GK != kGateHead ? 1 : 0;
            const __nv_bfloat16 *gr = log_alpha + (GK != kGateHead ? trow * dkin + c0 : trow),
                                *kr = k + trow * dkin + c0, *qr = q + trow * dkin + c0;
            const bool has_gate = GK != kGateHead || log_alpha != nullptr;
            // raw inputs: the 1 / L2 norms of the whole q and k rows
            float nk = 1.f, nq = 1.f;
            if constexpr (GK == kRawInputs) {
                const uint4 *k8 = reinterpret_cast<const uint4 *>(k + trow * dkin);
                const uint4 *q8 = reinterpret_cast<const uint4 *>(q + trow * dkin);
                float sk = 0.f, sq = 0.f;
                for (int c8 = 0; c8 < dkin / 8; ++c8) {
                    float f[8];
                    unpack8(k8[c8], f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) sk = fmaf(f[i], f[i], sk);
                    unpack8(q8[c8], f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) sq = fmaf(f[i], f[i], sq);
                }
                nk = rsqrtf(sk + kNormEps);
                nq = rsqrtf(sq + kNormEps);
            }
            float pk = 0.f, pq = 0.f, kq = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                // key channels past the input's width: no decay, zero key and query
                float lg = kin ? __bfloat162float(gr[i * gstride]) : 0.f;
                if constexpr (GK == kRawInputs) lg = kin ? log_sigmoid(lg) : 0.f;
                const float a = has_gate ? expf(lg) : 1.f, kk = kin ? __bfloat162float(kr[i]) * nk : 0.f,
                            qq = kin ? __bfloat162float(qr[i]) * nq : 0.f;
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
            const float u = jv ? beta_of<GK>(beta, trow) * (__bfloat162float(v[trow * DV + j]) - spk) : 0.f;
            if (qd == 0 && jv) out[trow * DV + j] = from_f32<TO>(fmaf(u, skq, spq));
            if (kin) {
#pragma unroll
                for (int i = 0; i < 32; ++i) S[i] = fmaf(__bfloat162float(kr[i]) * nk, u, S[i]);
            }
            tc::named_sync(kBarRole, kRoleThreads);
        }
        return write_state_operand();
    };

    uint32_t ph1 = 0, ph2 = 0;
    int t = 0;   // chunk number within this chain
    bool stop = false;
    for (int pr = kc; pr < sched.npairs && !stop; pr += sched.nchain) {
        const PairInfo pi = pair_info(sched, pr);
        h = pi.h;
        const size_t state_base = ((size_t)pi.n * H + h) * dkin * DV + (size_t)c0 * DV + j;
#pragma unroll
        for (int i = 0; i < 32; ++i) S[i] = (init_state && jv && kin) ? init_state[state_base + (size_t)i * DV] : 0.f;
        tc::tc_fence_before();
        bool force_exact = tc::named_sync_or(kBarRole, kRoleThreads, write_state_operand());
        bool have_image = false;   // the previous chunk's last barrier already covered this chunk's image
        for (int c = 0; c < pi.nchunks; ++c, ++t) {
            const int s = t % SM::kSlots, b = t & 1;
            const int64_t tok0 = pi.tok0(c);
            const int L = pi.len(c);
            const uint8_t *slot = sm + s * SM::kSlotBytes;
            const uint32_t sslot = sbase + s * SM::kSlotBytes;
            if (!have_image &&
                !role_wait(&bars.full[s], (t / SM::kSlots) & 1, leader, kBarRole, kRoleThreads, abort_flag)) {
                stop = true;
                break;
            }
            have_image = false;
            if (*abort_flag) {
                stop = true;
                break;
            }
            // chunk t is out of the ring (the copy has completed): its slot may take a later image
            if (leader) tc::st_relaxed_gpu(sched.consumed + kc, t + 1);
            const bool flagged = *reinterpret_cast<const volatile int *>(slot + I::kFlag) != 0;
            if (leader) {
                // the output warps have read D1^T[b] of chunk t - 2
                bool ok = t < 2 || tc::mbar_wait(&bars.d1_free[b], ((t >> 1) - 1) & 1, abort_flag);
                if (ok && !flagged) {
                    tc::tc_fence_after();
                    // ---- D1^T[b] = S^T [-W ; Qg]^T ----
                    constexpr uint32_t id1 = tc::make_idesc(128, 128, tc::kF16, false, false);
#pragma unroll
                    for (int kk = 0; kk < kDK / 16; ++kk)
                        tc::mma_f16_ta(tmem + kTmD1 + b * 128, tmem + kTmS + kk * 8,
                                       desc_kmajor(sslot + I::kA1, 128, kk), id1, kk > 0);
                    tc::mma_commit(&bars.mma1);
                }
                if (flagged) {
                    bars.outmode[b] = 0;   // no MMAs, no tensor output
                    tc::mbar_arrive(&bars.outq[b]);
                }
            }
            if (!flagged) {
                // while MMA1 runs: D2^T = S^T Diag(gamma) in fp32, which MMA2 then accumulates onto
                // (D2^T was last read by the previous chunk's state update)
                {
                    const float4 *gam4 = reinterpret_cast<const float4 *>(slot + I::kGam) + c0 / 4;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint32_t u[16];
#pragma unroll
                        for (int i4 = 0; i4 < 4; ++i4) {
                            const float4 gg = gam4[4 * h2 + i4];
                            const int i = 16 * h2 + 4 * i4;
                            u[4 * i4] = __float_as_uint(gg.x * S[i]);
                            u[4 * i4 + 1] = __float_as_uint(gg.y * S[i + 1]);
                            u[4 * i4 + 2] = __float_as_uint(gg.z * S[i + 2]);
                            u[4 * i4 + 3] = __float_as_uint(gg.w * S[i + 3]);
                        }
                        tc::tmem_st16(tmem + tl + kTmD2 + c0 + 16 * h2, u);
                    }
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                }
                // every state warp waits for MMA1 itself (no barrier round); a timeout is shared through
                // the barrier after the U~ epilogue
                if (!tc::mbar_wait(&bars.mma1, ph1, abort_flag)) *reinterpret_cast<volatile int *>(&bars.fail1) = 1;
                tc::tc_fence_after();
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
                            unpack8_h(*reinterpret_cast<const uint4 *>(slot + I::kUT + tile_chunk(j, 2 * qd + h2, DV)),
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
                if (mybad) *reinterpret_cast<volatile int *>(&bars.ovf_ut) = t + 1;
                tc::named_sync(kBarRole, kRoleThreads);
                const bool bad = *reinterpret_cast<volatile int *>(&bars.ovf_ut) == t + 1;
                if (*reinterpret_cast<volatile int *>(&bars.fail1)) {
                    stop = true;
                    break;
                }
                if (leader) {
                    tc::tc_fence_after();
                    // ---- D2^T += U~^T Kd;  D1^T[b][:, 64:128] += U~^T P^T ----
                    constexpr uint32_t id2 = tc::make_idesc(128, 128, tc::kF16, false, true);
                    constexpr uint32_t id3 = tc::make_idesc(128, kChunk, tc::kF16, false, false);
#pragma unroll
                    for (int kk = 0; kk < kChunk / 16; ++kk)
                        tc::mma_f16_ta(tmem + kTmD2, tmem + kTmUt + kk * 8, desc_mnmajor(sslot + I::kKd, kChunk, kk),
                                       id2, true);
                    tc::mma_commit(&bars.mma2);
#pragma unroll
                    for (int kk = 0; kk < kChunk / 16; ++kk)
                        tc::mma_f16_ta(tmem + kTmD1 + b * 128 + 64, tmem + kTmUt + kk * 8,
                                       desc_kmajor(sslot + I::kP, kChunk, kk), id3, true);
                    tc::mma_commit(&bars.mma3[b]);
                    bars.outmode[b] = bad ? 1 : 2;   // MMAs issued; O^T is the output unless evaluated exactly
                    tc::mbar_arrive(&bars.outq[b]);
                }
                if (!tc::mbar_wait(&bars.mma2, ph2, abort_flag)) *reinterpret_cast<volatile int *>(&bars.fail2) = 1;
                tc::tc_fence_after();
                ph2 ^= 1u;
                if (!bad) {
                    // ---- S^T = D2^T = S^T Diag(gamma) + U~^T Kd ----
                    tc::tmem_ld32(tmem + tl + kTmD2 + c0, S);
                    tc::tmem_ld_wait();
                    const bool big = write_state_operand();
                    tc::tc_fence_before();
                    if (big) *reinterpret_cast<volatile int *>(&bars.ovf_st) = t + 1;
                    // the next chunk's image (two chunks ahead, normally landed long ago): the leader waits
                    // for it here, so that this barrier serves both
                    if (c + 1 < pi.nchunks) {
                        if (leader) tc::mbar_wait(&bars.full[(t + 1) % SM::kSlots], ((t + 1) / SM::kSlots) & 1,
                                                  abort_flag);
                        have_image = true;
                    }
                    tc::named_sync(kBarRole, kRoleThreads);
                    tc::tc_fence_after();
                    force_exact = *reinterpret_cast<volatile int *>(&bars.ovf_st) == t + 1;
                    if (*reinterpret_cast<volatile int *>(&bars.fail2)) {
                        stop = true;
                        break;
                    }
                    continue;
                }
            }
            // exact path: the chunk's decays exceed the rebasing range, or an fp16 value overflowed
            const bool big = exact_chunk(tok0, L);
            tc::tc_fence_before();
            force_exact = tc::named_sync_or(kBarRole, kRoleThreads, big);
            if (*reinterpret_cast<volatile int *>(&bars.fail2)) {
                stop = true;
                break;
            }
        }
        if (!stop && final_state && *abort_flag == 0 && jv && kin) {
#pragma unroll
            for (int i = 0; i < 32; ++i) final_state[state_base + (size_t)i * DV] = S[i];
        }
    }
    if (leader) drain_mma(&bars.fin, 0);
}

// ====================================== kernel and launch ==========================================
template <int DV, typename TO, int GK>
__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_tc_kernel(const __grid_constant__ RowMaps maps, const __grid_constant__ ChunkSched sched,
                    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                    const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ log_alpha,
                    const __nv_bfloat16 *__restrict__ beta, const float *init_state, TO *__restrict__ out,
                    float *final_state) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ ChunkBars bars;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ int s_tmax;

    const int tid = threadIdx.x, warp = tid >> 5;
    const bool is_chain = static_cast<int>(blockIdx.x) < sched.nchain;
    if (tid == 0) {
        if (!is_chain) s_tmax = chain_tmax(sched);
        for (int i = 0; i < 2; ++i) tc::mbar_init(&bars.full[i], 1);
        tc::mbar_init(&bars.mma1, 1);
        tc::mbar_init(&bars.mma2, 1);
        tc::mbar_init(&bars.mma3[0], 1);
        tc::mbar_init(&bars.mma3[1], 1);
        tc::mbar_init(&bars.outq[0], 1);
        tc::mbar_init(&bars.outq[1], 1);
        tc::mbar_init(&bars.d1_free[0], kThreads / 32 - kRoleWarps);
        tc::mbar_init(&bars.d1_free[1], kThreads / 32 - kRoleWarps);
        tc::mbar_init(&bars.m_ap, 1);
        tc::mbar_init(&bars.m_wu, 1);
        tc::mbar_init(&bars.staged, 1);
        tc::mbar_init(&bars.staging_free, 1);
        tc::mbar_init(&bars.raw_full, 2);
        tc::mbar_init(&bars.raw_free, 1);
        tc::mbar_init(&bars.fin, 1);
        tc::fence_mbar_init();
        abort_flag = 0;
        bars.fail1 = 0;
        bars.fail2 = 0;
        bars.ovf_ut = 0;
        bars.ovf_st = 0;
    }
    const uint32_t ncols = is_chain ? kTmChainCols : kTmPrepCols;
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base_sh, ncols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    ChunkCtx cx;
    cx.sm = sm;
    cx.sbase = tc::smem_u32(sm);
    cx.tmem = tmem_base_sh;
    cx.abort_flag = &abort_flag;
    if (is_chain)
        chain_role<DV, TO, GK>(cx, bars, sched, blockIdx.x, maps, q, k, v, log_alpha, beta, init_state, out,
                               final_state);
    else
        prep_role<DV, GK>(cx, bars, sched, blockIdx.x - sched.nchain, s_tmax, maps, log_alpha, beta);

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(cx.tmem, ncols);
}

// Workspace tables of the schedule: zeroes the ring flags and, for packed sequences, writes the
// longest-first order of the sequences (ties by index), so that long sequences start first.
__global__ void __launch_bounds__(256) kda_chunk_sched_kernel(const int32_t *__restrict__ cu, int num_seqs,
                                                              int32_t *order, int *flags, int nflags) {
    for (int i = threadIdx.x; i < nflags; i += blockDim.x) flags[i] = 0;
    if (!order) return;
    for (int n = threadIdx.x; n < num_seqs; n += blockDim.x) {
        const int ln = cu[n + 1] - cu[n];
        int rank = 0;
        for (int m = 0; m < num_seqs; ++m) {
            const int lm = cu[m + 1] - cu[m];
            rank += (lm > ln) || (lm == ln && m < n);
        }
        order[rank] = n;
    }
}

// Grid split for npairs (sequence, head) pairs on nsm SMs: at most a quarter of the SMs (and 64)
// run chains, a pair each per wave; the rest produce chunk images.
struct ChunkGrid {
    int nchain, nprod;
};
inline ChunkGrid chunk_grid(int64_t npairs, int nsm) {
    ChunkGrid g;
    int cap = nsm / 4;
    cap = cap < 1 ? 1 : (cap > 64 ? 64 : cap);
    const int64_t waves = (npairs + cap - 1) / cap;
    g.nchain = static_cast<int>((npairs + waves - 1) / waves);
    g.nprod = nsm - g.nchain;
    return g;
}
constexpr int kRing = 12;                // ring slots per chain (workspace variant)
constexpr int kMinRing = 3;
constexpr int kMaxChains = 64;
// sequence order (4 KB), then the ready flags, the consumed counters and the abort word
constexpr size_t kFlagsBytes = 4096 + (size_t)(kMaxChains * kRing + kMaxChains + 1) * 4;
template <int DV> constexpr size_t ring_stride() { return Img<DV>::kStride; }
inline size_t img_stride(int DV) { return DV == 64 ? Img<64>::kStride : Img<128>::kStride; }
inline size_t flags_region_bytes() { return (kFlagsBytes + 1023) / 1024 * 1024; }

// Bytes of global workspace kda_chunk_fwd needs on the tensor-core path: the schedule tables and a
// ring of kRing chunk images for each chain (at most kMaxChains chains, whatever the SM count).
inline size_t chunk_tc_workspace_bytes(int64_t pairs, int DV) {
    const int64_t chains = pairs < kMaxChains ? pairs : kMaxChains;
    return flags_region_bytes() + static_cast<size_t>(chains) * kRing * img_stride(DV);
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

// SM count of the current device (cached per device).
inline int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    static int cache[64] = {};
    if (dev < 0 || dev >= 64) return 0;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

// Testing hook of the chunk kernel: the producer item whose image is never published (-1: none)
// and the limit of the waits on the ring flags.  Process-wide, read at each launch.
struct ChunkFault {
    int skip_item = -1;
    uint64_t flag_wait_ns = tc::kFlagWaitNs;
};
inline ChunkFault &chunk_fault() {
    static ChunkFault f;
    return f;
}

// Launches the schedule-table kernel and the chunk kernel.  `ws_bytes` bounds the ring depth: the
// workspace holds the schedule tables and nchain rings of `ring` images (kMinRing <= ring <= kRing).
template <int DV, typename TO, int GK>
cudaError_t launch_chunk_tc_dv(const void *q, const void *k, const void *v, const void *la, const void *beta,
                               const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H,
                               int DKIN, int C, void *out, float *final_state, void *workspace, size_t ws_bytes,
                               cudaStream_t stream) {
    if (C < 1 || C > kChunk || (DKIN != 64 && DKIN != kDK)) return cudaErrorInvalidValue;
    auto kern = kda_chunk_tc_kernel<DV, TO, GK>;
    const int smem = chunk_smem_bytes<DV>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int N = cu ? num_seqs : B;
    const int64_t npairs = (int64_t)N * H;
    if (npairs <= 0) return cudaSuccess;
    const int nsm = device_sm_count();
    if (nsm < 2) return cudaErrorInvalidDevice;
    const ChunkGrid grid = chunk_grid(npairs, nsm);
    const size_t flags = flags_region_bytes();
    if (ws_bytes < flags) return cudaErrorInvalidValue;
    int64_t ring = static_cast<int64_t>((ws_bytes - flags) / ((size_t)grid.nchain * Img<DV>::kStride));
    if (ring > kRing) ring = kRing;
    if (ring < kMinRing) return cudaErrorInvalidValue;

    RowMaps maps;
    memset(&maps, 0, sizeof(maps));
    const int64_t tokens = (int64_t)B * T;
    if (tokens > 0) {   // with no tokens no chunk is loaded and the maps stay unused
        if ((GK != kGateHead && !encode_row_map(&maps.g, la, DKIN, H, tokens)) ||
            !encode_row_map(&maps.k, k, DKIN, H, tokens) ||
            !encode_row_map(&maps.q, q, DKIN, H, tokens) || !encode_row_map(&maps.v, v, DV, H, tokens) ||
            !encode_row_map(&maps.o, out, DV, H, tokens, 64,
                            sizeof(TO) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                            static_cast<int>(sizeof(TO))))
            return cudaErrorInvalidValue;
    }
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    ChunkSched sched;
    sched.npairs = static_cast<int>(npairs);
    sched.nchain = grid.nchain;
    sched.nprod = grid.nprod;
    sched.ring = static_cast<int>(ring);
    sched.H = H;
    sched.T = T;
    sched.C = C;
    sched.dk = DKIN;
    sched.cu = cu;
    const bool sorted = cu && num_seqs <= kLongestFirstMaxSeqs;
    sched.order = sorted ? reinterpret_cast<const int32_t *>(ws) : nullptr;
    sched.ready = reinterpret_cast<int *>(ws + 4096);
    sched.consumed = sched.ready + grid.nchain * sched.ring;
    sched.rings = ws + flags;
    sched.fw.abort_all = sched.consumed + grid.nchain;
    sched.fw.limit_ns = chunk_fault().flag_wait_ns;
    sched.skip_item = chunk_fault().skip_item;
    const int nflags = grid.nchain * sched.ring + grid.nchain + 1;
    kda_chunk_sched_kernel<<<1, 256, 0, stream>>>(cu, num_seqs, sorted ? reinterpret_cast<int32_t *>(ws) : nullptr,
                                                  sched.ready, nflags);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // every CTA must be resident at once (chains and producers wait on one another)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(grid.nchain + grid.nprod));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, kern, maps, sched, static_cast<const __nv_bfloat16 *>(q),
                              static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v),
                              static_cast<const __nv_bfloat16 *>(la), static_cast<const __nv_bfloat16 *>(beta),
                              init_state, static_cast<TO *>(out), final_state);
}

// `la`: log_alpha [tokens][H][d_k] (kGateChannel), the per-head log_g [tokens][H] or null
// (kGateHead), or the gate's pre-activation [tokens][H][d_k] (kRawInputs, with raw q, k, beta).
template <typename TO>
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const void *la, const void *beta,
                            const float *init_state, const int32_t *cu, int num_seqs, int B, int T, int H, int DKIN,
                            int DV, int C, void *out, float *final_state, void *workspace, size_t ws_bytes,
                            cudaStream_t stream, int gate = kGateChannel) {
#define KDA_CHUNK_TC_CASE(DVV, GKK)                                                                          \
    if (DV == DVV && gate == GKK)                                                                            \
        return launch_chunk_tc_dv<DVV, TO, GKK>(q, k, v, la, beta, init_state, cu, num_seqs, B, T, H, DKIN, C, out, \
                                                final_state, workspace, ws_bytes, stream);
    KDA_CHUNK_TC_CASE(64, kGateChannel)
    KDA_CHUNK_TC_CASE(128, kGateChannel)
    KDA_CHUNK_TC_CASE(64, kGateHead)
    KDA_CHUNK_TC_CASE(128, kGateHead)
    KDA_CHUNK_TC_CASE(64, kRawInputs)
    KDA_CHUNK_TC_CASE(128, kRawInputs)
#undef KDA_CHUNK_TC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace kda
