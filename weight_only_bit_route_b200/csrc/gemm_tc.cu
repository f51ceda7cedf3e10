// Grouped GEMM on the 5th-generation tensor cores (tcgen05), every batch size.
//
// Per expert e with n_e routed rows, gate/up computes
//     G = X_e Wg_e^T, U = X_e Wu_e^T, h = bf16(silu(G) * U)      (K = H)
// and down computes
//     Y = w * (Hp_e Wd_e^T)                                         (K = F)
// with the 4-bit weights turned into MMA operands inside the kernel
// ("Step-5-Preview-Int4-g128", Recipe; "Step-5-Preview-NVFP4-Local", Format).
//
// Tiles are swapped: weights are the M = 128 operand and tokens the N operand,
// because an expert sees few tokens (about 47 at 2048 tokens).  A tile is
// (expert, m-tile of 128 weight rows, n-tile of token rows: up to 64 for
// gate/up and 128 for down, 128 for "wide" gate/up tiles, 16 for "narrow"
// decode tiles, 5 tokens on the 8-bit path).  A persistent CTA per SM builds
// the tile list on the device from expert_offsets; warp 0 takes the CTA's
// tiles (in a blocked order, or from an atomic counter when the launch hands
// tiles out dynamically), computes their coordinates once and queues them for
// the other roles.
//
// Warp roles inside a CTA (16 warps):
//   warp 0      TMA producer of the weight stream: per stage, 2D tensor
//               copies of 128 rows x 128 bytes (K = 256 of packed 4-bit
//               weights, or K = 64 of BF16) per matrix, 128-byte swizzled,
//               plus the NVFP4 block scales of those rows.  int4 scales are
//               one bulk copy per tile, since all groups of the tile's rows
//               are contiguous.
//   warp 1      producer of the activation operand: per stage, TMA boxes of
//               the tile's rows, 128-byte swizzled (the K-major layout the MMA
//               descriptors read); the box height comes from one of several
//               tensor maps, matching the tile's rows (8-bit path: 16 digit
//               rows per box, and the tile's row records by bulk copy).
//   warp 2      allocates tensor memory and issues tcgen05.mma from one lane
//               (8-bit int4: warps 2 and 3 take alternate steps).
// The single-issue roles run warp-uniform loops and elect one lane to issue,
// which keeps the instruction operands in uniform registers.  The MMA
// pipeline steps in K = 128 (8-bit path: K = 256 for gate/up, 512 for down;
// W4A4: 256) and commits once per step, to one barrier of a ring of 16
// ("stage done"): a tcgen05.commit costs as much issue time as several MMAs,
// so every role that waits for a step to finish (the activation producer, the
// dequantisation warps, the BF16 weight producer, the small-batch epilogue)
// waits on that one barrier.  A parity wait only tells a phase from the one
// before it: every waiter either sees all phases of a barrier in order or
// first waits for something that orders it after the previous phase.
//   warps 4-7   epilogue: tcgen05.ld of the accumulators, SwiGLU or the
//               routing weight, bf16 stores.  Warp w reads TMEM lanes
//               32*(w%4) to 32*(w%4)+31.
//   warps 8-15  dequantisation (16-bit paths).  Each thread owns one weight
//               row of the tile.  It turns packed weights into exact f16
//               pairs in registers (int4: q s 2^k with a power of two per
//               weight row; NVFP4: e2m1 * e4m3) and writes them to tensor
//               memory with tcgen05.st; the MMA reads its A operand from
//               there, so dequantised weights never pass through shared
//               memory.  On the 8-bit path the warps only unpack nibbles into
//               bytes, in two groups of four that take alternate weight
//               stages.  On the W4A4 path warps 8-11 arrange the block scale
//               factors for tcgen05.cp and the MMA reads both operands from
//               shared memory.
// BF16 weights (the shared expert) need no dequantisation: the MMA reads the
// TMA-staged weight tile from shared memory directly.
//
// Tensor memory (512 columns): accumulator buffers first (two of 128 columns
// on the 16-bit paths, so the epilogue of one tile overlaps the main loop of
// the next; gate at +0 and up at +64 or +128), A stages after them.  The
// 8-bit path accumulates per step: its small accumulator buffers take
// [0, 128) and the A stages [128, 512).
//
// int4 words: one mask per nibble pair places the nibbles (j, j+4) of a packed
// word into one f16 pair, so the A operand holds the K elements of each group
// of 8 in the order 0,4,1,5,2,6,3,7 (8-bit path: 0,2,4,6,1,3,5,7); the
// activation pre-pass stores its rows in the same order.  A dot product does
// not depend on the order of its terms.
//
// Every wait is bounded (about 2 s).  On expiry the kernel records
// MOE_ERR_TIMEOUT and stops issuing work.  It then waits, again bounded, for
// the copies and MMAs it has in flight, frees its tensor memory and returns.
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "moe_internal.cuh"
#include "nvfp4_block.cuh"
#include "tc_ptx.cuh"

namespace moe {

constexpr int G_BM = 128;
constexpr int G_THREADS = 512;
constexpr int G_DQ_WARPS = 8;
constexpr int G_EPI_WARPS = 4;

// int4 with small token tiles (8-bit MMA): the dequantisation only unpacks
// each nibble u into a byte (two logic ops per 4 weights) and the tensor
// cores run kind::i8 (u8 weights x s8 activations, exact s32 sums, K = 32 per
// instruction).  The pre-pass writes each activation row as a 24-bit fixed
// point X = x * 2^c (c per row, |X| < 2^22) in three signed 8-bit digits,
// X = 65536 d2 + 256 d1 + d0, one B operand row per digit (token j's digits
// are rows 3j, 3j+1, 3j+2 of the tile: five tokens fill N = 16).  An MMA step
// covers K = 256; each of its two scale groups accumulates from zero into its
// own columns.  The epilogue warps combine the digit sums, subtract
// 8 * sum(X) over the group (the u - 8 offset) and fold scale * value into
// fp32 totals.  The group scale and the offset leave
// the per-weight work, and the accumulation itself is exact.  Internal
// format value.
constexpr int FMT_INT4_I8 = 3;
// NVFP4 W4A4 on the block-scaled FP4 tensor cores: weights and activations
// both E2M1 with E4M3 scales per 16, tcgen05.mma.kind::mxf4nvf4 with
// scale_vec::4X.  A (weights) and B (the quantised activations) are read from
// shared memory as stored, K = 64 per instruction; the scale factors go to
// tensor memory by tcgen05.cp.  Internal format value.
constexpr int FMT_NVFP4_A4 = 4;
constexpr int G_SF_RING = 4;                 // A4: scale-factor slots (shared and tensor memory)

// NW: tile width class.  1 (wide): gate/up tiles of up to 128 token rows
// instead of 64, for batches whose experts hold many rows: each dequantised
// weight then serves twice the tokens.  The 4-bit formats keep a single
// accumulator buffer of 256 columns (gate, up) and two A stages; BF16 (no A
// stages) keeps two buffers.  2 (narrow, BF16 and NVFP4 16-bit): at most 16
// token rows per tile, for decode batches (an expert holds at most one row per
// token): the activation stages shrink to 2 KB per K 64, and shared memory
// goes to weight stages in flight instead.
template <int FMT, bool GU, int NW = 0>
struct GCfg {
    static constexpr bool kI8 = FMT == FMT_INT4_I8;
    static constexpr bool kA4 = FMT == FMT_NVFP4_A4;
    static constexpr bool kInt4 = FMT == MOE_FMT_INT4_G128 || kI8;
    static constexpr bool kTmemA = FMT != MOE_FMT_BF16 && !kA4;     // A dequantised into tensor memory
    static constexpr bool kPacked = kTmemA || kA4;                    // 4-bit weight stages (128 B = K 256 per row)
    static constexpr bool kWide = NW == 1 && GU && !kI8;
    static constexpr bool kNarrow = NW == 2 && !kI8;
    static constexpr int kNMat = GU ? 2 : 1;
    static constexpr int kNMax = kI8 ? 5 : (kNarrow ? 16 : (GU ? (kWide ? 128 : 64) : 128));   // token rows per tile
    static constexpr int kUpCol = kWide ? 128 : 64;                 // 16-bit paths: up accumulator within a buffer
    // K per MMA step: 8-bit down steps are K = 512, so that the per-step fixed cost of the
    // issuer and the unpack warps covers 32 KB of weights, as a gate/up step does
    static constexpr int kSK = kI8 ? (GU ? 256 : 512) : (kA4 ? 256 : 128);
    static constexpr int kGroups = kSK / 128;                       // i8: scale groups per MMA stage
    static constexpr int kAccCols = kI8 ? kGroups * kNMat * 16 : (kWide ? 256 : 128);   // one accumulator buffer
    // Tensor memory: accumulators in [0, kABase), A stages in [kABase, 512).  The
    // 8-bit path keeps few small accumulators and gives the A ring the room
    // (its dequantise -> MMA -> free cycle is long against a step).
    static constexpr int kAccBufs = kI8 ? 128 / kAccCols : (kWide && kPacked ? 1 : (kWide ? 2 : 256 / kAccCols));
    static constexpr int kABase = kAccBufs * kAccCols;
    static constexpr int kMmaK = kI8 ? 32 : (kA4 ? 64 : 16);        // K per MMA instruction
    static constexpr int kPkK = kPacked ? (kI8 ? kSK : 256) : 128;  // K per weight stage
    static constexpr int kBoxes = kPacked ? kPkK / 256 : 2;         // 128-byte-wide TMA boxes per matrix and stage
    static constexpr int kMatBytes = kPacked ? G_BM * kPkK / 2 : G_BM * 256;   // one matrix of a weight stage
    static constexpr int kNvScBytes = (FMT == MOE_FMT_NVFP4 || kA4) ? G_BM * 16 : 0;
    static constexpr int kPkStageBytes = kNMat * (kMatBytes + kNvScBytes);
    static constexpr int kPkMax = 12;                               // weight stages: as many as fit, up to this
    static constexpr int kScStages = kI8 ? G_EPI_WARPS : G_DQ_WARPS;     // readers of the int4 scale buffer
    static constexpr int kBAtom = (kI8 ? 16 : kNMax) * 128;         // 128 bytes of K for every B row
    static constexpr int kBAtoms = kI8 ? kSK / 128 : (kA4 ? 1 : 2); // 128-byte K slices per B stage
    static constexpr int kBScBytes = kA4 ? kNMax * 16 : 0;          // A4: the B rows' raw scale factors
    static constexpr int kBStageBytes = kBAtoms * kBAtom + kBScBytes;
    // A4: per step the scale factors of kNMat weight tiles and the B tile, as 4 chunks (K 64 each)
    // of 512 bytes apiece in shared memory, and 4 tensor-memory columns per chunk
    static constexpr int kSfChunks = kA4 ? (kNMat + 1) * 4 : 0;
    static constexpr int kSfSlotBytes = kSfChunks * 512;
    static constexpr int kSfSlotCols = kSfChunks * 4;
    // i8 stages are small: cover the copy latency; wide stages are large: fit shared memory
    static constexpr int kBStages = kI8 ? (GU ? 6 : 4) : (kWide ? (kTmemA ? 3 : 2) : (kNarrow ? 6 : 4));
    static constexpr int kAColsK = kI8 ? kSK / 4 : 64;              // TMEM columns of one matrix's A stage
    static constexpr int kAStageCols = kNMat * kAColsK;
    static constexpr int kAStages = kTmemA ? (512 - kABase) / kAStageCols : 1;   // (BF16, A4: none used)
    static constexpr int kAPerPk = kPkK / kSK;                      // A stages per weight stage (2, or 1 for i8)
    static constexpr int kChunkCols = 16;                           // 16-bit paths: TMEM columns of one packed chunk
    static constexpr int kDqArrivals = kI8 ? G_DQ_WARPS / 2 : G_DQ_WARPS;  // warps that fill one stage
    static constexpr bool kMmaF16 = FMT == MOE_FMT_NVFP4 || FMT == MOE_FMT_INT4_G128;   // f16 operands
    // warps that read the tile queue: activation producer, MMA issuer(s), epilogue, and the
    // scale-factor (A4) or dequantisation / unpacking warps
    static constexpr int kQReaders = 1 + (kI8 ? 2 : 1) + G_EPI_WARPS + (kA4 ? 4 : (kTmemA ? G_DQ_WARPS : 0));
    static_assert(kABase <= 512 && (!kTmemA || kAStages >= 2), "tensor memory layout");
    // the 8-bit path's two MMA issuers take alternate steps: even B and accumulator rings give each
    // the slots it alone waits on, so it sees every phase of them in order; an issuer's accumulator
    // wait covers the other issuer's A stages as long as there are no more buffers than A stages
    static_assert(!kI8 || (kBStages % 2 == 0 && kAccBufs % 2 == 0 && kAccBufs <= kAStages),
                  "8-bit rings");
    static_assert(!kA4 || kABase + G_SF_RING * kSfSlotCols <= 512, "A4 scale-factor ring");
};

constexpr int G_DONE = 16;                                          // "stage done" barrier ring
constexpr int G_TQ = 16;                                            // tile queue: tile ids the producer hands out
constexpr int G_SC_MAX = 8;                                         // int4 scale buffers (one tile each)
constexpr int G_KSPLIT_MAX = 8;                                     // split-K slices summed inside the GEMM

constexpr int G_NB_MAPS = 8;                                        // box heights 16, 32, ..., 128

struct GArgs {
    CUtensorMap tm_p0, tm_p1;        // packed (or BF16) weights of gate (or down) and up
    CUtensorMap tm_s0, tm_s1;        // NVFP4 block scales
    CUtensorMap tm_b[G_NB_MAPS];     // activation operand rows, box height 16*(i+1) (8-bit int4: [0], digit rows)
    CUtensorMap tm_bs[G_NB_MAPS];    // A4: the activation rows' scale factors, box height 16*(i+1)
    const uint8_t* sc0;              // int4 scales (bf16), bulk-copied per tile
    const uint8_t* sc1;
    const float* g0;                 // NVFP4 per-expert global scales
    const float* g1;
    const int32_t* offsets;
    const int32_t* row_slot;
    const float* topk_w;             // down: routing weight by slot (nullable)
    const float* act_scale;          // NVFP4: activation row scale, by GEMM row
    __nv_bfloat16* out;
    int32_t* status;
    float* partial;                  // split-K: fp32 partial sums [ksplit][nmat][rows][out_dim]
    const float* zsum;               // 8-bit int4: per row, 8 * sum of the fixed-point values of each group, each
                                     // group's 2^-c, the row factor: [rows][2 * zst + 4]
    int E, out_dim, in_dim;
    int ksplit, rows;                // K slices per (m-tile, n-tile); activation rows of the problem
    int* tile_cnt;                   // split-K: zeroed arrival counters, four per (m-tile, n-tile); the last
                                     // epilogue warp of each quarter sums the slices (else a kernel does)
    int* sched;                      // null: tile blockIdx.x + i * gridDim.x; else {next, done}: tiles handed out by
                                     // an atomic counter, zero on entry, left at zero by the last CTA
    int early;                       // the kernel before is this GEMM's pre-pass, which lets it start once that has
                                     // waited for its own predecessor: only the roles that read the pre-pass's
                                     // output (activation producer, epilogue) wait for it; the tile list and the
                                     // weight stream start at once
    int npk;                         // weight stages in the shared-memory ring (2 .. kPkMax)
    int nsc;                         // int4 scale buffers (2 .. G_SC_MAX)
};

// ---------------------------------------------------------------------------
// Dequantisation of one 16-byte chunk of packed weights (32 weights) into 16
// bf16/f16 pairs.  int4: pair order within each 8, sc = bf16 scale bits.
// NVFP4: natural order, sc = two E4M3 bytes (K 0-15, K 16-31 of the chunk).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void g_dq_int4(const uint4 w, uint32_t s2, uint32_t s16, uint32_t (&o)[16]) {
    // s2 = {s', s'} and s16 = {s'/16, s'/16} in f16, s' = the group scale times the row's power of
    // two.  A mask puts nibbles (p, p+4) of a word into the mantissas of 1024.0 (p even, values
    // 1024 + u) or of 1024.0 with the nibble four bits up (p odd, 1024 + 16 u): subtracting 1032 or
    // 1152 gives q or 16 q exactly, and one multiply by s' or s'/16 gives q s' exactly (at most
    // 11 significant bits, in f16's normal range by the choice of the row's power of two).
    const __half2 hs = *reinterpret_cast<const __half2*>(&s2);
    const __half2 hs16 = *reinterpret_cast<const __half2*>(&s16);
    const __half2 off0 = __floats2half2_rn(1032.f, 1032.f), off1 = __floats2half2_rn(1152.f, 1152.f);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const uint32_t t = ws[j] >> 8;
        uint32_t v0 = (ws[j] & 0x000F000Fu) | 0x64006400u;      // nibbles 0, 4
        uint32_t v1 = (ws[j] & 0x00F000F0u) | 0x64006400u;      // nibbles 1, 5 (x 16)
        uint32_t v2 = (t & 0x000F000Fu) | 0x64006400u;          // nibbles 2, 6
        uint32_t v3 = (t & 0x00F000F0u) | 0x64006400u;          // nibbles 3, 7 (x 16)
        __half2 h0 = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&v0), off0), hs);
        __half2 h1 = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&v1), off1), hs16);
        __half2 h2 = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&v2), off0), hs);
        __half2 h3 = __hmul2(__hsub2(*reinterpret_cast<__half2*>(&v3), off1), hs16);
        o[j * 4 + 0] = *reinterpret_cast<uint32_t*>(&h0);
        o[j * 4 + 1] = *reinterpret_cast<uint32_t*>(&h1);
        o[j * 4 + 2] = *reinterpret_cast<uint32_t*>(&h2);
        o[j * 4 + 3] = *reinterpret_cast<uint32_t*>(&h3);
    }
}
// The power of two k that puts a row's largest int4 group scale m in [2^11, 2^12): then every
// q s 2^k (|q| <= 8) stays below 2^15 and is exact in f16 down to scales 2^25 below m.
__device__ __forceinline__ int g_int4_row_shift(float m) {
    if (!(m > 0.f)) return 0;
    int e = 0;
    frexpf(m, &e);                                       // m = f 2^e, f in [0.5, 1)
    return min(60, max(-24, 12 - e));
}
// the f16 pair {s 2^k, s 2^k} and {s 2^k / 16, ...} of a bf16 group scale
__device__ __forceinline__ void g_int4_scale_pair(uint32_t sbf16, float fk, uint32_t& s2, uint32_t& s16) {
    const float sv = __uint_as_float(sbf16 << 16) * fk;
    __half2 a = __float2half2_rn(sv), b = __float2half2_rn(sv * 0.0625f);
    s2 = *reinterpret_cast<uint32_t*>(&a);
    s16 = *reinterpret_cast<uint32_t*>(&b);
}
__device__ __forceinline__ void g_dq_nvfp4(const uint4 w, uint32_t sc2, uint32_t (&o)[16]) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        uint32_t sv = g_e4m3_f16x2((sc2 >> (8 * (j >> 1))) & 0xffu);
        const __half2 s2 = *reinterpret_cast<__half2*>(&sv);
        uint32_t hv[4];
        g_e2m1x8_f16x2(ws[j], hv);                       // the word's four bytes, no shifts
#pragma unroll
        for (int b = 0; b < 4; b++) {
            __half2 h = __hmul2(*reinterpret_cast<__half2*>(&hv[b]), s2);       // exact
            o[j * 4 + b] = *reinterpret_cast<uint32_t*>(&h);
        }
    }
}

// 8-bit int4: the nibbles of each word as bytes, even nibbles first: the K
// order within every 8 weights becomes 0, 2, 4, 6, 1, 3, 5, 7.  One 16-byte
// chunk gives 8 words, at o[OFF .. OFF + 7].
template <int OFF>
__device__ __forceinline__ void g_dq_int4_i8(const uint4 w, uint32_t (&o)[16]) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        o[OFF + 2 * j] = ws[j] & 0x0F0F0F0Fu;
        o[OFF + 2 * j + 1] = (ws[j] >> 4) & 0x0F0F0F0Fu;
    }
}

struct GTile { int e, m0, n0, nval, bn, ebase, ks, kbase, mn; };

// Bytes of the per-expert tile table at the start of the dynamic shared memory (16 per expert),
// rounded so the stage rings after it stay 1024-byte aligned.
__host__ __device__ inline uint32_t g_tbl_bytes(int E) { return (uint32_t(E) * 16u + 1023u) & ~1023u; }

// ---------------------------------------------------------------------------
// Kernel
// ---------------------------------------------------------------------------
template <int I, int N, class F>
__device__ __forceinline__ void g_static_for(F&& f) {
    if constexpr (I < N) {
        f(std::integral_constant<int, I>{});
        g_static_for<I + 1, N>(f);
    }
}

template <int FMT, bool GU, int NW>
__global__ void __launch_bounds__(G_THREADS, 1) tc_grouped_gemm(const __grid_constant__ GArgs a) {
    using C = GCfg<FMT, GU, NW>;
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ __align__(8) uint64_t pk_full[C::kPkMax], pk_empty[C::kPkMax];
    __shared__ __align__(8) uint64_t b_full[C::kBStages], a_full[C::kAStages], done[G_DONE];
    __shared__ __align__(8) uint64_t sc_full[G_SC_MAX], sc_empty[G_SC_MAX];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], drain;
    __shared__ __align__(8) uint64_t hold_bar;        // failure testing: a barrier nothing completes
    __shared__ __align__(8) uint64_t sf_full[G_SF_RING];   // A4: a step's scale-factor chunks are in place
    __shared__ __align__(8) uint64_t tq_full[G_TQ], tq_empty[G_TQ];   // tile queue
    __shared__ int s_tq[G_TQ];
    __shared__ GTile s_tqt[G_TQ];                    // the queued tiles' coordinates (computed once, by warp 0)
    __shared__ int s_first;
    __shared__ int s_hold;
    __shared__ uint32_t s_tmem;
    __shared__ int s_wsum[G_THREADS / 32], s_wt[G_THREADS / 32];
    __shared__ int s_nact, s_total;
    __shared__ volatile GAbort s_ab;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int MT = a.out_dim / G_BM;
    const int in_dim = a.in_dim;
    const int ksplit = a.ksplit;                                    // K slices (BF16 split-K), else 1
    const int kc = in_dim / ksplit;                                 // K of one tile
    const int KS = kc / C::kSK;                                     // MMA stages per tile
    const int NPS = kc / C::kPkK;                                   // weight stages per tile
    const int ngroups = in_dim / 128;
    const uint32_t sc_mat_bytes = uint32_t(G_BM * ngroups * 2);
    const int zst = ((ngroups + 3) & ~3);                           // i8: groups per row record, rounded to 4
    const int zrs = 2 * zst + 4;                                    // i8: row record (floats)
    // one scale buffer: the int4 scales of the tile's rows (per matrix), then
    // (i8) the group sums of the tile's tokens
    const uint32_t sc_buf_bytes = C::kNMat * sc_mat_bytes + (C::kI8 ? uint32_t(C::kNMax * zrs * 4) : 0u);
    const uint32_t NPK = uint32_t(a.npk);                          // weight stages in the ring
    const int NSC = a.nsc;                                          // int4 scale buffers, one tile each

    if (tid == 0) {
        for (int s = 0; s < a.npk; s++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&pk_full[s])));
            if (C::kTmemA)     // BF16 weight stages are freed through the "stage done" ring
                asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(g_smem(&pk_empty[s])), "r"(C::kDqArrivals));
        }
        for (int s = 0; s < C::kBStages; s++)   // i8: one asynchronous arrival per lane of the copying warp
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&b_full[s])));
        for (int s = 0; s < C::kAStages; s++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(g_smem(&a_full[s])), "r"(C::kDqArrivals));
        for (int s = 0; s < G_DONE; s++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&done[s])));
        for (int s = 0; s < a.nsc; s++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(g_smem(&sc_full[s])), "r"(C::kI8 ? 2 : 1));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(g_smem(&sc_empty[s])), "r"(C::kScStages));
        }
        for (int s = 0; s < 2; s++)          // (at most two buffers on the 16-bit paths)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&acc_full[s])));
        for (int s = 0; s < C::kAccBufs; s++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(g_smem(&acc_empty[s])), "r"(G_EPI_WARPS));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(g_smem(&drain)), "r"(C::kI8 ? 2 : 1));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&hold_bar)));
        for (int s = 0; s < G_SF_RING; s++)       // A4: one arrival per scale-factor warp
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(g_smem(&sf_full[s])), "r"(4));
        for (int s = 0; s < G_TQ; s++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(g_smem(&tq_full[s])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(g_smem(&tq_empty[s])), "r"(C::kQReaders));
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_ab.flag = 0;
        s_ab.limit_ns = G_WAIT_NS;
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(g_smem(&s_tmem)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (!a.early) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == 0) {                                   // published by the __syncthreads below
        s_ab.limit_ns = g_limit_from(a.status);
        s_hold = g_hold_from(a.status);
    }

    // Tile list: per active expert {expert, first tile, first row, rows}, in dynamic shared memory
    // ahead of the stage rings (every role looks a tile up here, with no global load)
    uint8_t* dbase = smem + ((1024u - (g_smem(smem) & 1023u)) & 1023u);
    int4* tbl = reinterpret_cast<int4*>(dbase);
    {
        // this CTA's first tile: asked for now, its latency partly hidden behind the scan below (a CTA
        // that gets its SM late, behind another kernel, then holds no tile meanwhile)
        int first = int(blockIdx.x);
        if (tid == 0 && a.sched) first = atomicAdd(a.sched, 1);
        constexpr int PER = kMaxE / G_THREADS;
        int cnt[PER], nt[PER], eb[PER], ne[PER], local = 0, ltiles = 0;
#pragma unroll
        for (int i = 0; i < PER; i++) {
            const int e = tid * PER + i;
            eb[i] = (e < a.E) ? a.offsets[e] : 0;
            const int n = (e < a.E) ? a.offsets[e + 1] - eb[i] : 0;
            ne[i] = n;
            cnt[i] = n > 0;
            nt[i] = n > 0 ? ((n + C::kNMax - 1) / C::kNMax) * MT * ksplit : 0;
            local += cnt[i];
            ltiles += nt[i];
        }
        int v = local, w = ltiles;
        for (int o = 1; o < 32; o <<= 1) {
            const int n1 = __shfl_up_sync(0xffffffffu, v, o), n2 = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) { v += n1; w += n2; }
        }
        if (lane == 31) { s_wsum[warp] = v; s_wt[warp] = w; }
        g_fence_before();
        __syncthreads();
        g_fence_after();
        int base = 0, tbase = 0, tot = 0, ttot = 0;
        for (int q = 0; q < G_THREADS / 32; q++) {
            if (q < warp) { base += s_wsum[q]; tbase += s_wt[q]; }
            tot += s_wsum[q];
            ttot += s_wt[q];
        }
        int pos = base + v - local, tpos = tbase + w - ltiles;
#pragma unroll
        for (int i = 0; i < PER; i++)
            if (cnt[i]) { tbl[pos] = make_int4(tid * PER + i, tpos, eb[i], ne[i]); pos++; tpos += nt[i]; }
        if (tid == 0) { s_nact = tot; s_total = ttot; s_first = first; }
        __syncthreads();
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const uint32_t tmem = s_tmem;
    const int ntiles = s_total, nact = s_nact;
    uint8_t* pk = dbase + g_tbl_bytes(a.E);
    uint8_t* bring = pk + NPK * C::kPkStageBytes;
    uint8_t* scbuf = bring + C::kBStages * C::kBStageBytes;         // int4: NSC buffers of sc_buf_bytes
    uint8_t* sfring = scbuf;                                        // A4: G_SF_RING slots of kSfSlotBytes (no int4 buffers)

    auto tile_of = [&](int tile) {
        int lo = 0, hi = nact - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tbl[mid].y <= tile) lo = mid; else hi = mid - 1;
        }
        const int4 te = tbl[lo];
        GTile t;
        t.e = te.x;
        const int local = tile - te.y;
        t.ebase = te.z;
        const int n_e = te.w;
        if (ksplit == 1 && n_e <= C::kNMax) {
            // one n-tile, no K slices (every decode tile): the m-tile is the position, no divisions
            t.ks = 0;
            t.kbase = 0;
            t.mn = local;
            t.m0 = local * G_BM;
            t.n0 = 0;
            t.nval = n_e;
            t.bn = (n_e + 15) & ~15;
            return t;
        }
        const int ntile = (n_e + C::kNMax - 1) / C::kNMax;
        const int per = (n_e + ntile - 1) / ntile;                  // balanced rows per n-tile
        t.ks = local % ksplit;                                      // K slice fastest
        t.kbase = t.ks * kc;
        const int mn = local / ksplit;
        t.mn = mn;
        // Blocks of BN n-tiles x all MT m-tiles, about one wave of the grid: inside a block the
        // n-tiles of an m-tile are adjacent (CTAs running together share the weight tile through
        // L2) and every n-tile's activation rows are read by all MT m-tiles within the same wave,
        // so both operands come from DRAM about once per block instead of the activations once
        // per m-tile.
        const int BN = max(1, int(gridDim.x) / MT);
        const int blk = mn / (MT * BN);
        const int bnb = min(BN, ntile - blk * BN);               // n-tiles in this block
        const int idx = mn - blk * MT * BN;
        t.m0 = (idx / bnb) * G_BM;
        t.n0 = (blk * BN + idx % bnb) * per;
        t.nval = min(per, n_e - t.n0);
        t.bn = (t.nval + 15) & ~15;
        return t;
    };
    auto fail = [&]() {
        set_status(a.status, MOE_ERR_TIMEOUT);
        s_ab.flag = 1;
    };
    // Tile queue: warp 0 publishes, in order, every tile it starts and finally a value >= ntiles;
    // the other roles take the same sequence.  A reader sees every phase of each slot in order (it
    // took the slot's previous entry itself), and warp 0 reuses a slot only after all readers have
    // taken its previous entry.  A wait that runs out ends the reader's loop (>= ntiles).
    auto q_take = [&](uint32_t& qi, GTile& T) -> int {
        const uint32_t slot = qi % G_TQ;
        if (!g_wait_w(g_smem(&tq_full[slot]), (qi / G_TQ) & 1, &s_ab)) {
            fail();
            return ntiles;
        }
        const int v = *reinterpret_cast<volatile int*>(&s_tq[slot]);
        if (v < ntiles) T = s_tqt[slot];
        __syncwarp();
        if (lane == 0) g_arrive(g_smem(&tq_empty[slot]));
        qi++;
        return v;
    };

    if (warp == 0) {
        // ---------------- weight producer (whole warp, one lane issues) ----------------
        uint32_t pc = 0, qi = 0;
        int t = 0;
        // hand a tile (or the end, >= ntiles) to the other roles
        auto publish = [&](int tile, const GTile& T) -> bool {
            const uint32_t slot = qi % G_TQ;
            if (qi >= G_TQ && !g_wait_w(g_smem(&tq_empty[slot]), ((qi / G_TQ) - 1) & 1, &s_ab, 32)) {
                fail();
                return false;
            }
            if (lane == 0) {
                if (tile < ntiles) s_tqt[slot] = T;
                s_tq[slot] = tile;
                g_arrive(g_smem(&tq_full[slot]));
            }
            __syncwarp();
            qi++;
            return true;
        };
        // the tile's scales and weight stages
        auto produce = [&](const GTile& T) -> bool {
            const int row0 = T.e * a.out_dim + T.m0;
            if (C::kInt4) {
                const int b = t % NSC;
                if (t >= NSC && !g_wait_w(g_smem(&sc_empty[b]), ((t / NSC) - 1) & 1, &s_ab, 64)) {
                    fail();
                    return false;
                }
                const uint32_t bar = g_smem(&sc_full[b]);
                uint8_t* dst = scbuf + b * sc_buf_bytes;
                if (g_elect()) {         // (8-bit: the tokens' group sums come from the activation producer)
                    g_expect(bar, sc_mat_bytes * C::kNMat);
                    g_bulk(g_smem(dst), a.sc0 + size_t(row0) * ngroups * 2, sc_mat_bytes, bar);
                    if (GU) g_bulk(g_smem(dst + sc_mat_bytes), a.sc1 + size_t(row0) * ngroups * 2, sc_mat_bytes, bar);
                }
                __syncwarp();
            }
            t++;
            for (int ps = 0; ps < NPS; ps++, pc++) {
                const int s = pc % NPK;
                // 4-bit stages are freed by the dequantisation warps, BF16 ones by the MMA step
                // (A4 stages too: the MMA reads them from shared memory)
                if (pc >= NPK && !(C::kTmemA ? g_wait_w(g_smem(&pk_empty[s]), ((pc / NPK) - 1) & 1, &s_ab, 32)
                                             : g_wait_w(g_smem(&done[(pc - NPK) % G_DONE]), ((pc - NPK) / G_DONE) & 1,
                                                        &s_ab, 32))) {
                    fail();
                    return false;
                }
                const uint32_t bar = g_smem(&pk_full[s]);
                const uint32_t st = g_smem(pk + s * C::kPkStageBytes);
                if (g_elect()) {
                    g_expect(bar, C::kPkStageBytes);
                    if (C::kPacked) {
                        // 4-bit: 128 bytes of each row = K 256 per box, kBoxes boxes side by side
#pragma unroll
                        for (int h = 0; h < C::kBoxes; h++) {
                            const int x = T.kbase / 2 + ps * (C::kPkK / 2) + h * 128;
                            g_tma2d(st + h * (G_BM * 128), &a.tm_p0, x, row0, bar);
                            if (GU) g_tma2d(st + C::kMatBytes + h * (G_BM * 128), &a.tm_p1, x, row0, bar);
                        }
                        if (FMT == MOE_FMT_NVFP4 || C::kA4) {
                            const uint32_t ss = st + C::kNMat * C::kMatBytes;
                            g_tma2d(ss, &a.tm_s0, T.kbase / 16 + ps * 16, row0, bar);
                            if (GU) g_tma2d(ss + C::kNvScBytes, &a.tm_s1, T.kbase / 16 + ps * 16, row0, bar);
                        }
                    } else {
                        // BF16: two 64-element halves of K 128 per matrix
#pragma unroll
                        for (int h = 0; h < 2; h++) {
                            const int x = T.kbase + ps * 128 + h * 64;
                            g_tma2d(st + h * (G_BM * 128), &a.tm_p0, x, row0, bar);
                            if (GU) g_tma2d(st + C::kMatBytes + h * (G_BM * 128), &a.tm_p1, x, row0, bar);
                        }
                    }
                }
                __syncwarp();
            }
            return true;
        };
        // Dynamic order: lane 0 asks for a tile id one tile before the id is needed, into one of two
        // registers that the two halves of the loop below take turns with: an atomic under a full
        // weight stream takes microseconds (its reply queues behind this SM's incoming copies), and a
        // pending value must never be moved between registers, which would wait for it at once.
        int tile = s_first, fa = 0, fb = 0;
        if (lane == 0 && a.sched && tile < ntiles) fa = atomicAdd(a.sched, 1);
        GTile T{};
        while (!g_aborted(&s_ab)) {
            if (tile < ntiles) T = tile_of(tile);
            if (!publish(tile, T) || tile >= ntiles) break;
            if (lane == 0 && a.sched) fb = atomicAdd(a.sched, 1);
            if (!produce(T)) break;
            tile = a.sched ? __shfl_sync(0xffffffffu, fa, 0) : tile + int(gridDim.x);
            if (tile < ntiles) T = tile_of(tile);
            if (g_aborted(&s_ab) || !publish(tile, T) || tile >= ntiles) break;
            if (lane == 0 && a.sched) fa = atomicAdd(a.sched, 1);
            if (!produce(T)) break;
            tile = a.sched ? __shfl_sync(0xffffffffu, fb, 0) : tile + int(gridDim.x);
        }
        // the scheduler's counters: a CTA stops at its first id past the end, with one id after it
        // in flight; once that is back it counts itself done, and the last CTA to do so leaves both
        // counters at zero for the next launch.  (Reading fa and fb makes the lane wait for the one
        // in flight, so it is performed before the count; ids are never negative.)
        if (a.sched && lane == 0 && tile >= ntiles &&
            atomicAdd(a.sched + 1, (fa | fb) < 0 ? 2 : 1) == int(gridDim.x) - 1) {
            a.sched[0] = 0;
            a.sched[1] = 0;
        }
        // drain: every copy issued has landed before the CTA exits
        if (lane == 0) {
            const uint32_t first = pc > NPK ? pc - NPK : 0;
            for (uint32_t n = first; n < pc; n++) g_drain_wait(g_smem(&pk_full[n % NPK]), (n / NPK) & 1);
            if (C::kInt4)
                for (int n = t > NSC ? t - NSC : 0; n < t; n++) g_drain_wait(g_smem(&sc_full[n % NSC]), (n / NSC) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- activation producer (whole warp, one lane issues) ----------------
        // The activation rows come from the kernel before (the pre-pass): with an early start the
        // weight stream has been running since the prologue, and this role waits for them here.
        if (a.early) asm volatile("griddepcontrol.wait;" ::: "memory");
        uint32_t bc = 0;
        uint32_t qi = 0;
        int t = 0;
        bool ok = true;
        GTile T{};
        for (int tile = q_take(qi, T); tile < ntiles && ok && !g_aborted(&s_ab); tile = q_take(qi, T), t++) {
            const int row0 = (C::kI8 ? 3 : 1) * (T.ebase + T.n0);      // i8: three digit rows per token
            const CUtensorMap* map = &a.tm_b[C::kI8 ? 0 : T.bn / 16 - 1];
            if constexpr (C::kI8) {
                // the tile's tokens' group sums and factors, into the tile's scale buffer beside the
                // weight scales that warp 0 copies (sc_full takes both arrivals)
                const int b = t % NSC;
                if (t >= NSC && !g_wait_w(g_smem(&sc_empty[b]), ((t / NSC) - 1) & 1, &s_ab, 64)) {
                    fail();
                    ok = false;
                    break;
                }
                const uint32_t bar = g_smem(&sc_full[b]);
                const uint32_t zbytes = uint32_t(T.nval * zrs * 4);
                if (g_elect()) {
                    g_expect(bar, zbytes);
                    g_bulk(g_smem(scbuf + b * sc_buf_bytes + C::kNMat * sc_mat_bytes),
                           a.zsum + size_t(T.ebase + T.n0) * zrs, zbytes, bar);
                }
                __syncwarp();
            }
            for (int ks = 0; ks < KS; ks++, bc++) {
                const int s = bc % C::kBStages;
                if (bc >= uint32_t(C::kBStages) && !g_wait_w(g_smem(&done[(bc - C::kBStages) % G_DONE]),
                                                             ((bc - C::kBStages) / G_DONE) & 1, &s_ab, 32)) {
                    ok = false;
                    break;
                }
                const uint32_t bar = g_smem(&b_full[s]);
                const uint32_t st = g_smem(bring + s * C::kBStageBytes);
                if (g_elect()) {
                    if constexpr (C::kI8) {
                        // 16 digit rows (128-byte swizzled) per 128-byte K slice of the step; rows past the
                        // problem's last read as zero
                        g_expect(bar, uint32_t(C::kBStageBytes));
#pragma unroll
                        for (int h = 0; h < C::kBAtoms; h++)
                            g_tma2d(st + h * C::kBAtom, map, T.kbase + ks * C::kSK + h * 128, row0, bar);
                    } else if constexpr (C::kA4) {
                        // K 256 of packed E2M1 (128 bytes per row, swizzled) and the rows' 16 scale bytes
                        g_expect(bar, uint32_t(T.bn) * (128u + 16u));
                        g_tma2d(st, map, (T.kbase + ks * C::kSK) / 2, row0, bar);
                        g_tma2d(st + C::kBAtom, &a.tm_bs[T.bn / 16 - 1], (T.kbase + ks * C::kSK) / 16, row0, bar);
                    } else {
                        g_expect(bar, uint32_t(T.bn) * 256u);
                        g_tma2d(st, map, T.kbase + ks * C::kSK, row0, bar);
                        g_tma2d(st + C::kBAtom, map, T.kbase + ks * C::kSK + 64, row0, bar);
                    }
                }
                __syncwarp();
            }
            if (!ok) { fail(); break; }
        }
        if (lane == 0) {
            const uint32_t first = bc > uint32_t(C::kBStages) ? bc - C::kBStages : 0;
            for (uint32_t n = first; n < bc; n++) g_drain_wait(g_smem(&b_full[n % C::kBStages]), (n / C::kBStages) & 1);
        }
        __syncwarp();
    } else if (warp == 2 || (C::kI8 && warp == 3)) {
        // ---------------- MMA issuer (whole warp, one lane issues) ----------------
        // The 8-bit path has two issuers, warps 2 and 3, taking the even and odd
        // steps: its steps share no accumulator, and one issuing warp alone
        // cannot keep up with the weight stream (each step costs it about a
        // thousand cycles of serial work around eight or sixteen MMAs).
        const uint32_t n_iss = C::kI8 ? 2u : 1u, iss = uint32_t(warp - 2);
        // failure testing (moe_set_wait_hold): wait for a barrier that nothing completes, so the
        // bound runs out while the producers have copies in flight and the kernel takes its abort path
        if (s_hold && !g_wait_w(g_smem(&hold_bar), 0, &s_ab)) fail();
        uint32_t bc = 0, ac = 0, pc = 0;
        int t = 0;
        uint32_t qi = 0;
        GTile T{};
        for (int tile = q_take(qi, T); tile < ntiles && !g_aborted(&s_ab); tile = q_take(qi, T), t++) {
            const uint32_t idesc = C::kI8 ? g_idesc_i8(T.bn) : g_idesc(T.bn, C::kMmaF16);
            const int buf = C::kI8 ? 0 : t % C::kAccBufs;
            uint32_t d = tmem + buf * C::kAccCols;
            if (!C::kI8 && t >= C::kAccBufs &&
                !g_wait_w(g_smem(&acc_empty[buf]), ((t / C::kAccBufs) - 1) & 1, &s_ab)) {
                fail();
                break;
            }
            g_fence_after();
            bool ok = true;
            for (int ks = 0; ks < KS; ks++) {
                if (C::kI8 && bc % n_iss != iss) {      // the other issuer's step
                    bc++;
                    ac++;
                    continue;
                }
                const int sb = bc % C::kBStages, sa = ac % C::kAStages;
                if (C::kI8) {
                    // every step into the next accumulator buffer, freed by the epilogue.  This wait comes
                    // first: the two issuers take alternate steps and the A ring is odd, so the step that
                    // last filled A stage sa (ac - kAStages) was the other issuer's; the release of step
                    // bc - kAccBufs means the epilogue, which goes in order, has seen every earlier step,
                    // so that fill has landed and the parity wait on a_full below cannot pass a phase early
                    const int bi = bc % C::kAccBufs;
                    if (bc >= uint32_t(C::kAccBufs) &&
                        !g_wait_w(g_smem(&acc_empty[bi]), ((bc / C::kAccBufs) - 1) & 1, &s_ab)) { ok = false; break; }
                    d = tmem + bi * C::kAccCols;
                }
                if (!g_wait_w(g_smem(&b_full[sb]), (bc / C::kBStages) & 1, &s_ab)) { ok = false; break; }
                if (C::kTmemA) {
                    if (!g_wait_w(g_smem(&a_full[sa]), (ac / C::kAStages) & 1, &s_ab)) { ok = false; break; }
                } else {
                    if (!g_wait_w(g_smem(&pk_full[pc % NPK]), (pc / NPK) & 1, &s_ab)) { ok = false; break; }
                }
                if (C::kA4 && !g_wait_w(g_smem(&sf_full[bc % G_SF_RING]), (bc / G_SF_RING) & 1, &s_ab)) {
                    ok = false;
                    break;
                }
                g_fence_after();
                const uint32_t b0 = g_smem(bring + sb * C::kBStageBytes);
                const uint32_t at = tmem + C::kABase + sa * C::kAStageCols;
                const uint32_t a0 = g_smem(pk + (pc % NPK) * C::kPkStageBytes);
                if constexpr (C::kA4) {
                    // scale factors of this step into tensor-memory slot bc % G_SF_RING (A chunks of each
                    // matrix, then B's), then per K 64 one block-scaled MMA per matrix
                    const uint32_t slot = tmem + C::kABase + (bc % G_SF_RING) * C::kSfSlotCols;
                    const uint32_t sfs = g_smem(sfring + (bc % G_SF_RING) * C::kSfSlotBytes);
                    const uint32_t idesc4 = g_idesc_mxf4(T.bn);
                    if (g_elect()) {
#pragma unroll
                        for (int c = 0; c < C::kSfChunks; c++) g_cp_sf(slot + 4 * c, g_desc_sf(sfs + c * 512));
#pragma unroll
                        for (int k = 0; k < 4; k++) {
                            const uint64_t bd = g_desc(b0 + k * 32);
                            const uint32_t acc = (k > 0 || ks > 0) ? 1u : 0u;
                            const uint32_t sfb = slot + C::kNMat * 16 + 4 * k;
                            g_mma_mxf4(d, g_desc(a0 + k * 32), bd, idesc4, acc, slot + 4 * k, sfb);
                            if (GU) g_mma_mxf4(d + C::kUpCol, g_desc(a0 + C::kMatBytes + k * 32), bd, idesc4, acc,
                                               slot + 16 + 4 * k, sfb);
                        }
                        g_commit(g_smem(&done[bc % G_DONE]));
                    }
                } else if (g_elect()) {
#pragma unroll
                    for (int k = 0; k < C::kSK / C::kMmaK; k++) {
                        const uint64_t bd = g_desc(b0 + (k >> 2) * C::kBAtom + (k & 3) * 32);
                        if (C::kI8) {
                            // group k / 4 of the step into its own accumulator: gate at 16 g, up at 16 (kGroups + g)
                            const uint32_t acc = (k & 3) ? 1u : 0u;
                            const uint32_t dg = d + (k >> 2) * 16;
                            g_mma_ts_i8(dg, at + k * 8, bd, idesc, acc);
                            if (GU) g_mma_ts_i8(dg + C::kGroups * 16, at + C::kAColsK + k * 8, bd, idesc, acc);
                        } else if (C::kTmemA) {
                            const uint32_t acc = (k > 0 || ks > 0) ? 1u : 0u;
                            g_mma_ts(d, at + k * 8, bd, idesc, acc);
                            if (GU) g_mma_ts(d + C::kUpCol, at + C::kAColsK + k * 8, bd, idesc, acc);
                        } else {
                            const uint32_t acc = (k > 0 || ks > 0) ? 1u : 0u;
                            const uint32_t ak = a0 + (k >> 2) * (G_BM * 128) + (k & 3) * 32;
                            g_mma_ss(d, g_desc(ak), bd, idesc, acc);
                            if (GU) g_mma_ss(d + C::kUpCol, g_desc(ak + C::kMatBytes), bd, idesc, acc);
                        }
                    }
                    g_commit(g_smem(&done[bc % G_DONE]));
                }
                __syncwarp();
                bc++;
                if (C::kTmemA) ac++; else pc++;
            }
            if (!ok) { fail(); break; }
            if (!C::kI8 && g_elect()) g_commit(g_smem(&acc_full[buf]));
            __syncwarp();
        }
        // drain: every MMA issued has completed
        if (g_elect()) g_commit(g_smem(&drain));
        __syncwarp();
        if (lane == 0) g_drain_wait(g_smem(&drain), 0);
        __syncwarp();
    } else if (warp >= 4 && warp < 8 && C::kI8) {
        // ---------------- 8-bit int4 epilogue: fold every K = 128 step ----------------
        // Thread (warp w, lane l) owns weight row 32*(w%4) + l of the tile; lane
        // j < kNMax also holds token j's row factor.  A step holds kGroups scale
        // groups, each in its own 16 accumulator columns (gate, then up); token
        // j's digit sums are columns 3j (d2), 3j+1 (d1), 3j+2 (d0) of a group.
        if (a.early) asm volatile("griddepcontrol.wait;" ::: "memory");   // the pre-pass's row factors and sums
        const int q = warp & 3;
        const uint32_t lane_addr = uint32_t(q * 32) << 16;
        const int r = q * 32 + lane;
        uint32_t ac = 0;
        int t = 0;
        bool ok = true;
        uint32_t qi = 0;
        GTile T{};
        for (int tile = q_take(qi, T); tile < ntiles && ok && !g_aborted(&s_ab); tile = q_take(qi, T), t++) {
            const int f = T.m0 + r;
            const int rbase = T.ebase + T.n0;
            const bool live = lane < T.nval;
            const int b = t % NSC;
            if (!g_wait_w(g_smem(&sc_full[b]), (t / NSC) & 1, &s_ab, 64)) { ok = false; break; }
            const __nv_bfloat16* sc0 = reinterpret_cast<const __nv_bfloat16*>(scbuf + b * sc_buf_bytes) + r * ngroups;
            const __nv_bfloat16* sc1 = sc0 + G_BM * ngroups;
            const float* zs = reinterpret_cast<const float*>(scbuf + b * sc_buf_bytes + C::kNMat * sc_mat_bytes);
            // the token's row factor (the routing weight on down, 1 on gate/up) travels in its row record
            // (a global load from an SM under a full weight stream would take microseconds)
            const float rowf = live ? zs[lane * zrs + 2 * zst] : 1.f;
            float tg[C::kNMax], tu[C::kNMax];
#pragma unroll
            for (int j = 0; j < C::kNMax; j++) tg[j] = tu[j] = 0.f;
            for (int ks = 0; ks < KS; ks++, ac++) {
                const int bi = ac % C::kAccBufs;
                if (!g_wait_w(g_smem(&done[ac % G_DONE]), (ac / G_DONE) & 1, &s_ab)) { ok = false; break; }
                g_fence_after();
                uint32_t g[C::kGroups][16], u[C::kGroups][16];
                const uint32_t ab = tmem + lane_addr + bi * C::kAccCols;
#pragma unroll
                for (int gi = 0; gi < C::kGroups; gi++) {
                    g_ld16(ab + gi * 16, g[gi]);
                    if (GU) g_ld16(ab + (C::kGroups + gi) * 16, u[gi]);
                }
                g_ld_wait();
                g_fence_before();
                __syncwarp();
                if (lane == 0) g_arrive(g_smem(&acc_empty[bi]));
                // the step's kGroups scales of this row are adjacent: one 4- or 8-byte load per matrix
                const int grp0 = T.kbase / 128 + ks * C::kGroups;
                using SV = typename std::conditional<C::kGroups == 4, uint2, uint32_t>::type;
                const SV sv0 = *reinterpret_cast<const SV*>(sc0 + grp0);
                SV sv1{};
                if (GU) sv1 = *reinterpret_cast<const SV*>(sc1 + grp0);
                const uint32_t* s0w = reinterpret_cast<const uint32_t*>(&sv0);
                const uint32_t* s1w = reinterpret_cast<const uint32_t*>(&sv1);
#pragma unroll
                for (int gi = 0; gi < C::kGroups; gi++) {
                    const int grp = grp0 + gi;
                    const float s0 = __uint_as_float((s0w[gi >> 1] >> (16 * (gi & 1))) << 16);
                    const float s1 = GU ? __uint_as_float((s1w[gi >> 1] >> (16 * (gi & 1))) << 16) : 0.f;
#pragma unroll
                    for (int j = 0; j < C::kNMax; j++) {
                        if (j >= T.nval) break;                  // uniform: the tokens of this tile only
                        // the group's sum of u X less 8 sum X, times 2^-c of the group (exact), times the scale
                        const float zj = zs[j * zrs + grp], fj = zs[j * zrs + zst + grp];
                        const float vg = fmaf(float(int(g[gi][3 * j])), 65536.f,
                                              fmaf(float(int(g[gi][3 * j + 1])), 256.f, float(int(g[gi][3 * j + 2])))) - zj;
                        tg[j] = fmaf(s0, vg * fj, tg[j]);
                        if (GU) {
                            const float vu = fmaf(float(int(u[gi][3 * j])), 65536.f,
                                                  fmaf(float(int(u[gi][3 * j + 1])), 256.f, float(int(u[gi][3 * j + 2])))) - zj;
                            tu[j] = fmaf(s1, vu * fj, tu[j]);
                        }
                    }
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) g_arrive(g_smem(&sc_empty[b]));
#pragma unroll
            for (int j = 0; j < C::kNMax; j++) {
                const float fj = __shfl_sync(0xffffffffu, rowf, j);
                if (j < T.nval) {
                    float v;
                    if (GU) {
                        const float gg = tg[j] * fj, uu = tu[j] * fj;
                        v = gg / (1.0f + expf(-gg)) * uu;
                    } else {
                        v = tg[j] * fj;
                    }
                    a.out[size_t(rbase + j) * a.out_dim + f] = __float2bfloat16_rn(v);
                }
            }
        }
        if (!ok) fail();
    } else if (warp >= 4 && warp < 8) {
        // ---------------- epilogue ----------------
        if (a.early) asm volatile("griddepcontrol.wait;" ::: "memory");   // the pre-pass's row factors
        const int q = warp & 3;
        const uint32_t lane_addr = uint32_t(q * 32) << 16;
        int t = 0;
        uint32_t qi = 0;
        GTile T{};
        for (int tile = q_take(qi, T); tile < ntiles && !g_aborted(&s_ab); tile = q_take(qi, T), t++) {
            const int buf = t % C::kAccBufs;
            const int rbase = T.ebase + T.n0;
            // the factor of row c + j (activation row scale, routing weight) sits in lane j;
            // the loads of the first 16 rows' factors and of the global scales go out before the wait
            auto row_factor = [&](int c) {
                float v = 1.f;
                const int nn = c + (lane & 15);
                if (nn < T.nval) {
                    if (C::kMmaF16 || C::kA4) v = a.act_scale[rbase + nn];
                    // 4-bit formats: the pre-pass folded the routing weight into the row scale
                    if (!GU && a.topk_w && !(C::kMmaF16 || C::kA4)) v *= a.topk_w[a.row_slot[rbase + nn]];
                }
                return v;
            };
            float rowf0 = row_factor(0);
            float gsc = 1.f, usc = 1.f;
            if (FMT == MOE_FMT_NVFP4 || C::kA4) { gsc = a.g0[T.e]; if (GU) usc = a.g1[T.e]; }
            if (FMT == MOE_FMT_INT4_G128) {
                // undo the dequantisation's power of two of this weight row (gate and up separately)
                const int row = T.e * a.out_dim + T.m0 + q * 32 + lane;
                const int ng2 = a.in_dim / 256;                   // bf16 scale pairs per row
                float mg = 0.f, mu = 0.f;
                const uint32_t* s0r = reinterpret_cast<const uint32_t*>(a.sc0) + size_t(row) * ng2;
                const uint32_t* s1r = reinterpret_cast<const uint32_t*>(a.sc1) + size_t(row) * ng2;
                for (int g2 = 0; g2 < ng2; g2++) {
                    const uint32_t v = __ldg(s0r + g2);
                    mg = fmaxf(mg, fmaxf(fabsf(bf16_lo(v)), fabsf(bf16_hi(v))));
                    if (GU) {
                        const uint32_t w = __ldg(s1r + g2);
                        mu = fmaxf(mu, fmaxf(fabsf(bf16_lo(w)), fabsf(bf16_hi(w))));
                    }
                }
                gsc = ldexpf(1.f, -g_int4_row_shift(mg));
                if (GU) usc = ldexpf(1.f, -g_int4_row_shift(mu));
            }
            if (!g_wait_w(g_smem(&acc_full[buf]), (t / C::kAccBufs) & 1, &s_ab, 128)) { fail(); break; }
            g_fence_after();
            const int f = T.m0 + q * 32 + lane;
            const uint32_t acc0 = tmem + lane_addr + buf * C::kAccCols;
            for (int c = 0; c < T.bn; c += 16) {
                const float rowf = c == 0 ? rowf0 : row_factor(c);
                uint32_t g[16], u[16];
                g_ld16(acc0 + c, g);
                if (GU) g_ld16(acc0 + C::kUpCol + c, u);
                g_ld_wait();
                if (FMT == MOE_FMT_BF16 && ksplit > 1) {
                    // split-K: raw fp32 sums of this K slice; the tile's last slice (or a kernel) finishes the rows
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        if (c + j < T.nval) {
                            const size_t r = size_t(rbase + c + j);
                            a.partial[((size_t(T.ks) * C::kNMat) * a.rows + r) * a.out_dim + f] = __uint_as_float(g[j]);
                            if (GU)
                                a.partial[((size_t(T.ks) * C::kNMat + 1) * a.rows + r) * a.out_dim + f] = __uint_as_float(u[j]);
                        }
                    }
                    continue;
                }
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    const float fj = __shfl_sync(0xffffffffu, rowf, j);
                    if (c + j < T.nval) {
                        float v;
                        if (GU) {
                            const float gg = __uint_as_float(g[j]) * gsc * fj;
                            const float uu = __uint_as_float(u[j]) * usc * fj;
                            v = gg / (1.0f + expf(-gg)) * uu;
                        } else {
                            v = __uint_as_float(g[j]) * gsc * fj;
                        }
                        a.out[size_t(rbase + c + j) * a.out_dim + f] = __float2bfloat16_rn(v);
                    }
                }
            }
            g_fence_before();
            __syncwarp();
            if (lane == 0) g_arrive(g_smem(&acc_empty[buf]));
            if (FMT == MOE_FMT_BF16 && ksplit > 1 && a.tile_cnt) {
                // Per (tile, quarter of its rows): the epilogue warp that writes the last K slice of
                // its 32 rows sums all slices in slice order and writes the bf16 rows (E = 1: no
                // routing weight on gate/up, the slot weight on down).  Warps count separately, so
                // no warp ever waits for another here.
                __threadfence();
                __syncwarp();
                int last = 0;
                if (lane == 0) last = atomicAdd(&a.tile_cnt[T.mn * 4 + q], 1) == ksplit - 1;
                if (__shfl_sync(0xffffffffu, last, 0)) {
                    __threadfence();
                    const size_t plane = size_t(a.rows) * a.out_dim;
                    for (int j = 0; j < T.nval; j++) {
                        const size_t o = size_t(rbase + j) * a.out_dim + f;
                        // all slices' loads first (ksplit <= G_KSPLIT_MAX), then the sums in slice order
                        float pg[G_KSPLIT_MAX], pu[G_KSPLIT_MAX];
#pragma unroll
                        for (int k = 0; k < G_KSPLIT_MAX; k++) {
                            pg[k] = k < ksplit ? a.partial[(size_t(k) * C::kNMat) * plane + o] : 0.f;
                            pu[k] = (GU && k < ksplit) ? a.partial[(size_t(k) * C::kNMat + 1) * plane + o] : 0.f;
                        }
                        float gs = 0.f, us = 0.f;
#pragma unroll
                        for (int k = 0; k < G_KSPLIT_MAX; k++) {
                            if (k < ksplit) {
                                gs += pg[k];
                                us += pu[k];
                            }
                        }
                        float v;
                        if (GU) {
                            v = gs / (1.0f + expf(-gs)) * us;
                        } else {
                            const float w = a.topk_w ? a.topk_w[a.row_slot[rbase + j]] : 1.f;
                            v = w * gs;
                        }
                        a.out[o] = __float2bfloat16_rn(v);
                    }
                    if (lane == 0) a.tile_cnt[T.mn * 4 + q] = 0;          // ready for the next call
                }
            }
        }
    } else if (warp >= 8 && warp < 12 && C::kA4) {
        // ---------------- A4: scale factors into the MMA's chunk layout ----------------
        // Thread (warp w, lane l) takes row r = 32 (w % 4) + l of the step's weight tiles and of
        // its B tile.  A chunk (K 64: four 16-element blocks) of 128 rows is 512 bytes with the
        // four factors of row 32 m1 + m0 at 16 m0 + 4 m1; the factors of one chunk are one word
        // of the row's 16 raw bytes.  Rows past the tile's token rows read as zero.
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t at = 16u * uint32_t(r & 31) + 4u * uint32_t(r >> 5);
        uint32_t bc = 0;
        bool ok = true;
        uint32_t qi = 0;
        GTile T{};
        for (int tile = q_take(qi, T); tile < ntiles && ok && !g_aborted(&s_ab); tile = q_take(qi, T)) {
            for (int ks = 0; ks < KS; ks++, bc++) {
                if (!g_wait_w(g_smem(&pk_full[bc % NPK]), (bc / NPK) & 1, &s_ab) ||
                    !g_wait_w(g_smem(&b_full[bc % C::kBStages]), (bc / C::kBStages) & 1, &s_ab) ||
                    (bc >= uint32_t(G_SF_RING) && !g_wait_w(g_smem(&done[(bc - G_SF_RING) % G_DONE]),
                                                            ((bc - G_SF_RING) / G_DONE) & 1, &s_ab))) {
                    ok = false;
                    break;
                }
                const uint8_t* wsc = pk + (bc % NPK) * C::kPkStageBytes + C::kNMat * C::kMatBytes;
                const uint8_t* bsc = bring + (bc % C::kBStages) * C::kBStageBytes + C::kBAtom;
                uint8_t* slot = sfring + (bc % G_SF_RING) * C::kSfSlotBytes;
#pragma unroll
                for (int m = 0; m < C::kNMat; m++) {
                    const uint4 v = *reinterpret_cast<const uint4*>(wsc + m * C::kNvScBytes + r * 16);
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int c = 0; c < 4; c++) *reinterpret_cast<uint32_t*>(slot + (m * 4 + c) * 512 + at) = w4[c];
                }
                const uint4 v = r < T.bn ? *reinterpret_cast<const uint4*>(bsc + r * 16) : make_uint4(0, 0, 0, 0);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int c = 0; c < 4; c++) *reinterpret_cast<uint32_t*>(slot + (C::kNMat * 4 + c) * 512 + at) = w4[c];
                g_fence_proxy_async();                  // generic stores, read by tcgen05.cp
                __syncwarp();
                if (lane == 0) g_arrive(g_smem(&sf_full[bc % G_SF_RING]));
            }
        }
        if (!ok) fail();
    } else if (warp >= 8 && C::kI8) {
        // ---------------- 8-bit int4 unpacking ----------------
        // Two groups of four warps take alternate weight stages; a warp unpacks
        // its 32 rows of every matrix of the stage.  A warp learns that its
        // tensor-memory stores have landed only by waiting for all of them, so
        // one group's wait overlaps the other group's stage.  Pieces of 32
        // bytes of a row (two chunks, 16 TMEM columns) are software-pipelined:
        // the next piece is unpacked while the store of the current one is in
        // flight.
        constexpr int kPpm = C::kPkK / 64;             // 32-byte pieces of a row per matrix and stage
        constexpr int kPieces = C::kNMat * kPpm;
        constexpr int kNBuf = 4;
        const int q = warp & 3, grp = (warp - 8) >> 2;
        const int r = q * 32 + lane;
        const uint32_t lane_addr = uint32_t(q * 32) << 16;
        uint32_t pc = 0;
        bool ok = true;
        uint32_t qi = 0;
        GTile Tq{};
        for (int tile = q_take(qi, Tq); tile < ntiles && ok && !g_aborted(&s_ab); tile = q_take(qi, Tq)) {
            for (int ps = 0; ps < NPS; ps++, pc++) {
                if (int(pc & 1) != grp) continue;
                const int s = pc % NPK;
                // A stage sa is free once the MMA of step pc - kAStages has completed.  A parity wait
                // only tells a phase from the one before it, so a wait on pk_full[s] must come after the
                // stage's previous fill (step pc - NPK) has landed.  With an even ring that step was
                // this group's own; with an odd one it was the other group's, and the release of A stage
                // sa (every step up to pc - kAStages unpacked, NPK >= kAStages) comes first.
                const int sa = pc % C::kAStages;
                auto a_free = [&]() {
                    return pc < uint32_t(C::kAStages) ||
                           g_wait_w(g_smem(&done[(pc - C::kAStages) % G_DONE]), ((pc - C::kAStages) / G_DONE) & 1, &s_ab);
                };
                if (((NPK & 1) && !a_free()) || !g_wait_w(g_smem(&pk_full[s]), (pc / NPK) & 1, &s_ab)) {
                    ok = false;
                    break;
                }
                const uint8_t* st = pk + s * C::kPkStageBytes;
                uint32_t o[kNBuf][16];
                uint4 raw[2][2];                                // packed chunks, loaded one piece ahead
                auto load = [&](auto uc) {
                    // piece u: matrix m, 16-byte chunks c0 and c0 + 1 of the row, in TMA box c0 / 8
                    constexpr int u = decltype(uc)::value, m = u / kPpm, c0 = 2 * (u % kPpm);
                    const uint8_t* wt = st + m * C::kMatBytes + (c0 / 8) * (G_BM * 128);
                    raw[u & 1][0] = *reinterpret_cast<const uint4*>(wt + g_swz(r, c0 % 8));
                    raw[u & 1][1] = *reinterpret_cast<const uint4*>(wt + g_swz(r, c0 % 8 + 1));
                };
                auto unpack = [&](auto uc) {
                    constexpr int u = decltype(uc)::value;
                    g_dq_int4_i8<0>(raw[u & 1][0], o[u % kNBuf]);
                    g_dq_int4_i8<8>(raw[u & 1][1], o[u % kNBuf]);
                    if constexpr (u + 2 < kPieces) load(std::integral_constant<int, u + 2>{});
                };
                load(std::integral_constant<int, 0>{});
                if constexpr (kPieces > 1) load(std::integral_constant<int, 1>{});
                unpack(std::integral_constant<int, 0>{});
                if (!(NPK & 1) && !a_free()) {
                    ok = false;
                    break;
                }
                g_fence_after();
                const uint32_t a0 = tmem + lane_addr + C::kABase + sa * C::kAStageCols;
                g_static_for<0, kPieces>([&](auto uc) {
                    constexpr int u = decltype(uc)::value;
                    g_st16(a0 + (u / kPpm) * C::kAColsK + (u % kPpm) * 16, o[u % kNBuf]);
                    if constexpr (u + 1 < kPieces) unpack(std::integral_constant<int, u + 1>{});
                });
                g_st_wait();
                g_fence_before();
                __syncwarp();
                if (lane == 0) {
                    g_arrive(g_smem(&a_full[sa]));
                    g_arrive(g_smem(&pk_empty[s]));
                }
            }
        }
        if (!ok) fail();
    } else if (warp >= 8 && C::kTmemA) {
        // ---------------- dequantisation ----------------
        // A weight stage (K = 256, 8 chunks of 16 bytes per row) holds kAPerPk
        // A stages.  gate/up: this warp writes matrix hsel (all chunks of its
        // rows); down: it writes K half hsel of every A stage.  Chunks are
        // software-pipelined: the next one is dequantised while the tensor-
        // memory store of the current one is in flight.
        constexpr int kPer = (GU ? 8 : 4) / C::kAPerPk;    // my chunks per A stage
        constexpr int kChunks = C::kAPerPk * kPer;         // per weight stage
        constexpr int kNBuf = 4;
        const int q = warp & 3, hsel = (warp - 8) >> 2;
        const int r = q * 32 + lane;                   // weight row within the tile
        const uint32_t lane_addr = uint32_t(q * 32) << 16;
        const uint32_t colw = C::kABase + (GU ? hsel * C::kAColsK : hsel * kPer * C::kChunkCols);
        uint32_t pc = 0;
        int t = 0;
        bool ok = true;
        uint32_t qi = 0;
        GTile Tq{};
        for (int tile = q_take(qi, Tq); tile < ntiles && ok && !g_aborted(&s_ab); tile = q_take(qi, Tq), t++) {
            const uint8_t* scrow = nullptr;
            float fk = 1.f;                             // int4: 2^k of this weight row (the epilogue undoes it)
            if (FMT == MOE_FMT_INT4_G128) {
                const int b = t % NSC;
                if (!g_wait_w(g_smem(&sc_full[b]), (t / NSC) & 1, &s_ab)) { ok = false; break; }
                scrow = scbuf + b * sc_buf_bytes + (GU ? hsel * sc_mat_bytes : 0) + r * ngroups * 2;
                float m = 0.f;
                for (int g2 = 0; g2 < ngroups / 2; g2++) {
                    const uint32_t v = reinterpret_cast<const uint32_t*>(scrow)[g2];
                    m = fmaxf(m, fmaxf(fabsf(bf16_lo(v)), fabsf(bf16_hi(v))));
                }
                fk = ldexpf(1.f, g_int4_row_shift(m));
            }
            for (int ps = 0; ps < NPS && ok; ps++, pc++) {
                const int s = pc % NPK;
                if (!g_wait_w(g_smem(&pk_full[s]), (pc / NPK) & 1, &s_ab)) { ok = false; break; }
                const uint8_t* st = pk + s * C::kPkStageBytes;
                const uint8_t* wt = st + (GU ? hsel * C::kMatBytes : 0);
                uint32_t scw = 0;                      // int4: bf16 scales of groups 2ps (low) and 2ps+1 (high)
                uint4 nsc = make_uint4(0, 0, 0, 0);    // NVFP4: the 16 E4M3 scales of this row and stage
                if (FMT == MOE_FMT_INT4_G128) scw = *reinterpret_cast<const uint32_t*>(scrow + ps * 4);
                else if (FMT == MOE_FMT_NVFP4)
                    nsc = *reinterpret_cast<const uint4*>(st + C::kNMat * C::kMatBytes + (GU ? hsel * C::kNvScBytes : 0) +
                                                          r * 16);
                const uint32_t nscw[4] = {nsc.x, nsc.y, nsc.z, nsc.w};
                uint32_t s2[2] = {0u, 0u}, s16[2] = {0u, 0u};   // int4: f16 scale pairs of the two groups
                if (FMT == MOE_FMT_INT4_G128) {
                    g_int4_scale_pair(scw & 0xffffu, fk, s2[0], s16[0]);
                    g_int4_scale_pair(scw >> 16, fk, s2[1], s16[1]);
                }
                // Four register buffers in rotation: a buffer is rewritten three
                // chunks after its tensor-memory store was issued, so the store
                // has read it by then and the dequantisation does not stall.
                uint32_t o[kNBuf][16];
                // chunk index (16 bytes of this row in the weight stage) of my i-th chunk
                auto dq = [&](auto ic) {
                    constexpr int i = decltype(ic)::value, j = i / kPer, l = i % kPer;
                    const int c = (8 / C::kAPerPk) * j + (GU ? l : kPer * hsel + l);
                    const uint4 w = *reinterpret_cast<const uint4*>(wt + g_swz(r, c));
                    if constexpr (FMT == MOE_FMT_INT4_G128) {
                        g_dq_int4(w, s2[j], s16[j], o[i % kNBuf]);
                    } else if constexpr (FMT == MOE_FMT_NVFP4) {
                        // the two E4M3 scales of chunk c are bytes 2c and 2c+1
                        const uint32_t sw = GU ? nscw[2 * j + (l >> 1)] : (hsel ? nscw[2 * j + 1] : nscw[2 * j]);
                        g_dq_nvfp4(w, sw >> (16 * (GU ? (l & 1) : l)), o[i % kNBuf]);
                    }
                };
                int sa = 0;
                dq(std::integral_constant<int, 0>{});
                g_static_for<0, kChunks>([&](auto ic) {
                    constexpr int i = decltype(ic)::value, j = i / kPer, l = i % kPer;
                    if (!ok) return;
                    if (l == 0) {
                        const uint32_t acn = pc * C::kAPerPk + j;    // A stage index in this CTA's stream
                        sa = acn % C::kAStages;
                        if (acn >= uint32_t(C::kAStages) && !g_wait_w(g_smem(&done[(acn - C::kAStages) % G_DONE]),
                                                                      ((acn - C::kAStages) / G_DONE) & 1, &s_ab)) {
                            ok = false;
                            return;
                        }
                        g_fence_after();
                    }
                    g_st16(tmem + lane_addr + colw + sa * C::kAStageCols + l * C::kChunkCols, o[i % kNBuf]);
                    if constexpr (i + 1 < kChunks) dq(std::integral_constant<int, i + 1>{});
                    if (l == kPer - 1) {
                        g_st_wait();
                        g_fence_before();
                        __syncwarp();
                        if (lane == 0) g_arrive(g_smem(&a_full[sa]));
                    }
                });
                __syncwarp();
                if (lane == 0) g_arrive(g_smem(&pk_empty[s]));
            }
            if (!ok) break;
            if (FMT == MOE_FMT_INT4_G128) {
                __syncwarp();
                if (lane == 0) g_arrive(g_smem(&sc_empty[t % NSC]));
            }
        }
        if (!ok) fail();
    }

    g_fence_before();
    __syncthreads();
    g_fence_after();
    if (warp == 2) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

// ---------------------------------------------------------------------------
// Activation pre-pass: gather the GEMM's rows (row r reads activation row
// row_slot[r] / top_k when by_token, else row r) into the operand order:
//   mode 0: bf16 copy (BF16 weights);
//   mode 2: f16 times 2^-e in natural order (NVFP4 weights);
//   mode 3: f16 times 2^-e, pairs (0,4) (1,5) (2,6) (3,7) in every 8 (int4
//           weights, the order of their dequantised pairs);
//   mode 5: NVFP4 W4A4 activations: each row quantised with its expert's
//           input scale g (the row's expert found in offsets), codes and
//           block scales as stored, row scale g;
// with e the exponent that puts the row's largest |x| 2^-e in [2^13, 2^14):
// every bf16 value becomes an f16 exactly (bf16 has 8 significant bits, f16
// 11) unless it is 2^27 below the row's largest.  The row scale 2^e (times
// row_w[row_slot[row]] when given: the down projection's routing weight, a
// power of two times w being exact) goes to scale[row].  One warp per row.
// ---------------------------------------------------------------------------
template <bool F16>
__global__ void __launch_bounds__(256) g_prep(const __nv_bfloat16* __restrict__ src, int in_dim,
                                              const int32_t* __restrict__ row_slot, int top_k, int by_token,
                                              int rows, int mode, const float* __restrict__ row_w,
                                              uint16_t* __restrict__ dst, float* __restrict__ scale,
                                              const int32_t* __restrict__ offsets, int E,
                                              const float* __restrict__ in_scale, size_t sc_off) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the GEMM that reads these rows may start now (its weight stream needs nothing from here)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (row >= rows) return;
    const int srow = by_token ? row_slot[row] / top_k : row;
    const uint4* s = reinterpret_cast<const uint4*>(src + size_t(srow) * in_dim);
    uint4* d = reinterpret_cast<uint4*>(dst + size_t(row) * in_dim);
    const int n16 = in_dim / 8;
    if (mode == 0) {
        for (int i = lane; i < n16; i += 32) d[i] = s[i];
        return;
    }
    if (mode == 5) {
        // NVFP4 W4A4 on the FP4 tensor cores: the codes (two per byte, even element low) and the
        // E4M3 block scales as stored, [rows, in / 2] then [rows, in / 16] (dst + sc_off bytes)
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offsets[mid] <= row) lo = mid; else hi = mid - 1;
        }
        const float g = in_scale[lo];
        uint8_t* d8 = reinterpret_cast<uint8_t*>(dst) + size_t(row) * (in_dim / 2);
        uint8_t* sc8 = reinterpret_cast<uint8_t*>(dst) + sc_off + size_t(row) * (in_dim / 16);
        for (int b = lane; b < in_dim / 16; b += 32) {
            const uint4 v0 = s[2 * b], v1 = s[2 * b + 1];
            const float xf[16] = {act_lo<F16>(v0.x), act_hi<F16>(v0.x), act_lo<F16>(v0.y), act_hi<F16>(v0.y),
                                  act_lo<F16>(v0.z), act_hi<F16>(v0.z), act_lo<F16>(v0.w), act_hi<F16>(v0.w),
                                  act_lo<F16>(v1.x), act_hi<F16>(v1.x), act_lo<F16>(v1.y), act_hi<F16>(v1.y),
                                  act_lo<F16>(v1.z), act_hi<F16>(v1.z), act_lo<F16>(v1.w), act_hi<F16>(v1.w)};
            uint32_t bytes[8];
            sc8[b] = uint8_t(nv_quant_block16(xf, g, bytes));
            *reinterpret_cast<uint2*>(d8 + 8 * b) = make_uint2(bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24),
                                                              bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24));
        }
        if (lane == 0) scale[row] = row_w ? g * row_w[row_slot[row]] : g;
        return;
    }
    float amax = 0.f;
    for (int i = lane; i < n16; i += 32) {
        const uint4 v = s[i];
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(act_lo<F16>(v.x)), fabsf(act_hi<F16>(v.x))), fmaxf(fabsf(act_lo<F16>(v.y)), fabsf(act_hi<F16>(v.y)))));
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(act_lo<F16>(v.z)), fabsf(act_hi<F16>(v.z))), fmaxf(fabsf(act_lo<F16>(v.w)), fabsf(act_hi<F16>(v.w)))));
    }
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int e = 0;
    if (amax > 0.f && isfinite(amax)) {
        frexpf(amax, &e);                       // amax = f 2^ex, f in [0.5, 1): amax 2^-(ex-14) in [2^13, 2^14)
        e = max(e - 14, -100);
    }
    const float down = ldexpf(1.f, -e);
    for (int i = lane; i < n16; i += 32) {
        const uint4 v = s[i];
        __half2 h[4];
        h[0] = __floats2half2_rn(act_lo<F16>(v.x) * down, act_hi<F16>(v.x) * down);
        h[1] = __floats2half2_rn(act_lo<F16>(v.y) * down, act_hi<F16>(v.y) * down);
        h[2] = __floats2half2_rn(act_lo<F16>(v.z) * down, act_hi<F16>(v.z) * down);
        h[3] = __floats2half2_rn(act_lo<F16>(v.w) * down, act_hi<F16>(v.w) * down);
        uint4 o = *reinterpret_cast<uint4*>(h);
        if (mode == 3) {                        // (x0 x1)(x2 x3)(x4 x5)(x6 x7) -> (x0 x4)(x1 x5)(x2 x6)(x3 x7)
            const uint4 n = o;
            o.x = __byte_perm(n.x, n.z, 0x5410);
            o.y = __byte_perm(n.x, n.z, 0x7632);
            o.z = __byte_perm(n.y, n.w, 0x5410);
            o.w = __byte_perm(n.y, n.w, 0x7632);
        }
        d[i] = o;
    }
    if (lane == 0) scale[row] = row_w ? ldexpf(1.f, e) * row_w[row_slot[row]] : ldexpf(1.f, e);
}

// 8-bit int4 pre-pass: one CTA of 128 threads per GEMM row (gathered like
// g_prep).  Per scale group g of 128 elements, X = rint(x * 2^c), c the
// group's exponent that puts its max |X| in [2^21, 2^22), written as signed
// digits X = 65536 d2 + 256 d1 + d0 in int8 rows 3 row (d2), 3 row + 1 (d1),
// 3 row + 2 (d0) of dst, in the K order 0, 2, 4, 6, 1, 3, 5, 7 of every 8
// (the order of the unpacked weight bytes).  zf[row] is a record of 2 zst + 4
// floats: [g] = 8 * sum of X over group g (the u - 8 offset of the weights),
// [zst + g] = 2^-c of group g, [2 zst] = the row factor: row_w[row_slot[row]]
// when row_w is given (the down projection's routing weight), else 1 (also in
// scale[row]).  A group
// holding an infinity or a NaN has no fixed point: it records
// MOE_ERR_NONFINITE and gets a NaN factor, so its token's outputs are NaN (as
// a floating-point product with that row would be) instead of finite values
// made from meaningless digits.  The 16 threads of a half warp hold a group
// (8 elements each), so every exponent comes from a half-warp reduction.
constexpr int G_PREP_I8_THREADS = 128;
template <bool F16>
__global__ void __launch_bounds__(G_PREP_I8_THREADS) g_prep_i8(const __nv_bfloat16* __restrict__ src, int in_dim,
                                                               const int32_t* __restrict__ row_slot, int top_k,
                                                               int by_token, const float* __restrict__ row_w,
                                                               uint8_t* __restrict__ dst, float* __restrict__ scale,
                                                               float* __restrict__ zf, int32_t* status) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the GEMM that reads these rows may be placed on free SMs now; it waits for this grid
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const int slot = (by_token || row_w) ? row_slot[row] : 0;
    const float rw = (tid == 0 && row_w) ? row_w[slot] : 1.f;   // used last: its load goes out first
    const int srow = by_token ? slot / top_k : row;
    const uint4* s = reinterpret_cast<const uint4*>(src + size_t(srow) * in_dim);
    const int n16 = in_dim / 8, zst = ((in_dim / 128) + 3) & ~3;
    float* zrow = zf + size_t(row) * (2 * zst + 4);
    uint8_t* d8 = dst + size_t(row) * 3 * in_dim;
    // every chunk's load goes out before any is used (up to kPrepRegs chunks per thread)
    constexpr int kPrepRegs = 4;
    uint4 v[kPrepRegs];
#pragma unroll
    for (int j = 0; j < kPrepRegs; j++) {
        const int i = tid + j * G_PREP_I8_THREADS;
        v[j] = i < n16 ? s[i] : make_uint4(0, 0, 0, 0);
    }
    bool bad = false;
    auto emit = [&](const int i, const uint4 w) {
        const float xs[8] = {act_lo<F16>(w.x), act_lo<F16>(w.y), act_lo<F16>(w.z), act_lo<F16>(w.w),
                             act_hi<F16>(w.x), act_hi<F16>(w.y), act_hi<F16>(w.z), act_hi<F16>(w.w)};
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 8; e++) amax = fmaxf(amax, fabsf(xs[e]));
        for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const bool finite = isfinite(amax);             // amax is NaN or inf when any element is
        int ex = 0;
        if (finite) frexpf(amax, &ex);                  // amax < 2^ex
        const int c = (finite && amax > 0.f) ? min(22 - ex, 126) : 0;   // |x| 2^c < 2^22
        const float fc = ldexpf(1.f, c);                // a power of two: x * fc is exact
        int zs = 0;
        if (i < n16) {
            uint32_t p2[2] = {0u, 0u}, p1[2] = {0u, 0u}, p0[2] = {0u, 0u};
#pragma unroll
            for (int e = 0; e < 8; e++) {
                const int X = finite ? __float2int_rn(xs[e] * fc) : 0;
                zs += X;
                const int d0 = ((X + 128) & 255) - 128;          // signed digits in [-128, 127]
                const int X1 = (X - d0) >> 8;
                const int d1 = ((X1 + 128) & 255) - 128;
                const int d2 = (X1 - d1) >> 8;
                p0[e >> 2] |= uint32_t(d0 & 255) << (8 * (e & 3));
                p1[e >> 2] |= uint32_t(d1 & 255) << (8 * (e & 3));
                p2[e >> 2] |= uint32_t(d2 & 255) << (8 * (e & 3));
            }
            *reinterpret_cast<uint2*>(d8 + size_t(i) * 8) = make_uint2(p2[0], p2[1]);
            *reinterpret_cast<uint2*>(d8 + in_dim + size_t(i) * 8) = make_uint2(p1[0], p1[1]);
            *reinterpret_cast<uint2*>(d8 + 2 * size_t(in_dim) + size_t(i) * 8) = make_uint2(p0[0], p0[1]);
        }
        for (int o = 8; o > 0; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
        if ((lane & 15) == 0 && i < n16) {
            zrow[i / 16] = 8.f * float(zs);
            zrow[zst + i / 16] = finite ? 1.f / fc : __int_as_float(0x7fc00000);   // quiet NaN
            bad = bad || !finite;
        }
    };
#pragma unroll
    for (int j = 0; j < kPrepRegs; j++)
        if (j * G_PREP_I8_THREADS < n16) emit(tid + j * G_PREP_I8_THREADS, v[j]);     // uniform condition
    for (int i0 = kPrepRegs * G_PREP_I8_THREADS; i0 < n16; i0 += G_PREP_I8_THREADS) {
        const int i = i0 + tid;
        emit(i, i < n16 ? s[i] : make_uint4(0, 0, 0, 0));
    }
    if (bad) set_status(status, MOE_ERR_NONFINITE);
    if (tid == 0) {
        scale[row] = rw;
        zrow[2 * zst] = rw;                              // the row factor, also in the row record
    }
}

// ---------------------------------------------------------------------------
// Split-K finish: sums the K slices of every (row, feature) in slice order,
// then h = bf16(silu(g) * u) (gate/up) or y = bf16(w * d) (down, w the routing
// weight of the row's slot, 1 without routing weights).  Four features per thread.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) g_splitk_finish(const float* __restrict__ part, int ksplit, int nmat, int rows,
                                                       int out_dim, const float* __restrict__ topk_w,
                                                       const int32_t* __restrict__ row_slot,
                                                       __nv_bfloat16* __restrict__ out) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const size_t n4 = size_t(rows) * out_dim / 4;
    const size_t plane = size_t(rows) * out_dim;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += size_t(gridDim.x) * blockDim.x) {
        float4 g = make_float4(0.f, 0.f, 0.f, 0.f), u = g;
        for (int k = 0; k < ksplit; k++) {
            const float4 a = reinterpret_cast<const float4*>(part + (size_t(k) * nmat) * plane)[i];
            g.x += a.x; g.y += a.y; g.z += a.z; g.w += a.w;
            if (nmat == 2) {
                const float4 b = reinterpret_cast<const float4*>(part + (size_t(k) * nmat + 1) * plane)[i];
                u.x += b.x; u.y += b.y; u.z += b.z; u.w += b.w;
            }
        }
        float v[4];
        if (nmat == 2) {
            v[0] = g.x / (1.0f + expf(-g.x)) * u.x;
            v[1] = g.y / (1.0f + expf(-g.y)) * u.y;
            v[2] = g.z / (1.0f + expf(-g.z)) * u.z;
            v[3] = g.w / (1.0f + expf(-g.w)) * u.w;
        } else {
            const int r = int((i * 4) / out_dim);
            const float w = topk_w ? topk_w[row_slot[r]] : 1.f;
            v[0] = w * g.x; v[1] = w * g.y; v[2] = w * g.z; v[3] = w * g.w;
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]), hi = __floats2bfloat162_rn(v[2], v[3]);
        uint2 o;
        o.x = *reinterpret_cast<uint32_t*>(&lo);
        o.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>(out)[i] = o;
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int FMT, bool GU, int NW>
static size_t g_smem_bytes(int in_dim, int npk, int nsc, int E) {
    using C = GCfg<FMT, GU, NW>;
    size_t b = g_tbl_bytes(E) + size_t(npk) * C::kPkStageBytes + size_t(C::kBStages) * C::kBStageBytes + 1024;
    if (C::kInt4) b += size_t(nsc) * (C::kNMat * G_BM * (in_dim / 128) * 2 + (C::kI8 ? C::kNMax * (((in_dim / 128) + 3) & ~3) * 4 : 0));
    if (C::kA4) b += size_t(G_SF_RING) * C::kSfSlotBytes;
    return b;
}

template <int FMT, bool GU, int NW = 0>
static int g_launch(const GArgs& a, cudaStream_t s, int max_ctas, bool pdl) {
    using C = GCfg<FMT, GU, NW>;
    auto k = tc_grouped_gemm<FMT, GU, NW>;
    // per device: SM count, the opt-in shared memory left beside the kernel's static shared memory,
    // and the dynamic shared memory size granted so far (read once; raised only when a call needs more)
    struct DevInfo {
        std::once_flag once;
        int sms = 0;
        size_t room = 0;
        std::atomic<size_t> granted{0};
        int rc = MOE_ERR_CUDA;
    };
    static DevInfo info[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    DevInfo& di = info[dev];
    std::call_once(di.once, [&] {
        int optin = 0;
        cudaFuncAttributes fa{};
        if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, k) != cudaSuccess)
            return;
        di.room = size_t(optin) - std::min(size_t(optin), fa.sharedSizeBytes);
        di.rc = MOE_OK;
    });
    if (di.rc != MOE_OK) return di.rc;
    const int sms = di.sms;
    // The weight stream wants as many bytes in flight as shared memory holds.
    // The producer runs ahead by whole tiles only as far as free int4 scale
    // buffers allow, so those cover the ring's reach: one per tile it spans,
    // plus the tile being consumed.
    const size_t room = di.room;
    const int nps = std::max(1, (a.in_dim / a.ksplit) / C::kPkK);            // weight stages per tile
    int npk = C::kPkMax, nsc = 2;
    for (; npk >= 2; npk--) {
        nsc = C::kInt4 ? std::min(G_SC_MAX, std::max(2, (npk + nps - 1) / nps + 1)) : 2;
        if (g_smem_bytes<FMT, GU, NW>(a.in_dim, npk, nsc, a.E) <= room) break;
    }
    if (npk < 2) return MOE_ERR_UNSUPPORTED;
    GArgs args = a;
    args.npk = npk;
    args.nsc = nsc;
    const size_t smem = g_smem_bytes<FMT, GU, NW>(a.in_dim, npk, nsc, a.E);
    if (smem > di.granted.load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        size_t cur = di.granted.load(std::memory_order_acquire);
        while (cur < smem && !di.granted.compare_exchange_weak(cur, smem, std::memory_order_acq_rel)) {
        }
    }
    const int grid = max_ctas > 0 ? std::min(sms, max_ctas) : sms;
    if (pdl) return launch_pdl(k, dim3(grid), dim3(G_THREADS), smem, s, args) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    k<<<grid, G_THREADS, smem, s>>>(args);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

#define G_TRY(x)                       \
    do {                               \
        int _rc = (x);                 \
        if (_rc != MOE_OK) return _rc; \
    } while (0)

int launch_grouped_gemm(const GemvProblem& p, bool gateup, int rows, const GemmBuffers& buf, cudaStream_t s) {
    if (p.out_dim % G_BM || p.in_dim % 256 || p.E > kMaxE) return MOE_ERR_UNSUPPORTED;
    const int ksplit = buf.ksplit > 1 ? buf.ksplit : 1;
    if (ksplit > 1 && (p.fmt != MOE_FMT_BF16 || p.E != 1 || p.in_dim % (ksplit * 128) || !buf.partial ||
                       p.out_dim % 4))
        return MOE_ERR_UNSUPPORTED;
    if (p.fmt == MOE_FMT_INT4_G128 &&
        ((reinterpret_cast<uintptr_t>(p.s0) & 15u) || (gateup && (reinterpret_cast<uintptr_t>(p.s1) & 15u))))
        return MOE_ERR_INVALID_ARG;
    if (p.in_scale && p.fmt != MOE_FMT_NVFP4) return MOE_ERR_UNSUPPORTED;
    // fp16 activations enter through the pre-pass: the 4-bit formats only (BF16 reads its rows as they are)
    if (p.act_f16 && p.fmt == MOE_FMT_BF16) return MOE_ERR_UNSUPPORTED;
    if (rows <= 0) return MOE_OK;
    G_TRY(g_encoder());

    const int in = p.in_dim, out = p.out_dim, E = p.E;
    const bool nv = p.fmt == MOE_FMT_NVFP4, i4 = p.fmt == MOE_FMT_INT4_G128;
    const bool a4 = nv && p.in_scale != nullptr;                      // W4A4 on the FP4 tensor cores
    const size_t a4_sc_off = align256(size_t(rows) * (in / 2));     // A4: scale bytes after the codes
    // the 8-bit down GEMM steps in K = 512; other widths take the 16-bit int4 path
    const bool i8 = i4 && buf.i8 && (gateup || in % 512 == 0);
    if (i8 && (!buf.zbuf || !buf.scale_buf || !buf.act_buf || ksplit > 1)) return MOE_ERR_UNSUPPORTED;
    // activation operand rows [rows, in]: bf16 (f16 for NVFP4) in the kernel's order; 8-bit int4: three
    // int8 digit rows per row
    const void* bsrc = p.act;
    const float* ascale = nullptr;
    bool prep_launched = false;
    if (!buf.act_ready || nv || i4) {
        if (!buf.act_buf || ((nv || i4) && !buf.scale_buf)) return MOE_ERR_WORKSPACE;
        if (i8) {
            const float* row_w = gateup ? nullptr : p.topk_w;
            if (launch_pdl(p.act_f16 ? g_prep_i8<true> : g_prep_i8<false>, dim3(rows), dim3(G_PREP_I8_THREADS), 0, s,
                           p.act, in, p.row_slot, p.top_k,
                           p.act_by_token, row_w, reinterpret_cast<uint8_t*>(buf.act_buf), buf.scale_buf,
                           buf.zbuf, p.status) != cudaSuccess)
                return MOE_ERR_CUDA;
        } else {
            const int mode = a4 ? 5 : (nv ? 2 : (i4 ? 3 : 0));
            const float* row_w = ((nv || i4) && !gateup) ? p.topk_w : nullptr;   // folded into the row scale
            if (launch_pdl(p.act_f16 ? g_prep<true> : g_prep<false>, dim3((rows * 32 + 255) / 256), dim3(256), 0, s,
                           p.act, in, p.row_slot, p.top_k,
                           p.act_by_token, rows, mode, row_w, reinterpret_cast<uint16_t*>(buf.act_buf),
                           buf.scale_buf, p.offsets, p.E, p.in_scale, a4_sc_off) != cudaSuccess)
                return MOE_ERR_CUDA;
        }
        bsrc = buf.act_buf;
        ascale = buf.scale_buf;
        prep_launched = true;
    }

    GArgs a;
    memset(&a, 0, sizeof(a));
    const uint64_t wrows = uint64_t(E) * out;
    if (p.fmt == MOE_FMT_BF16) {
        G_TRY(g_map(&a.tm_p0, true, p.p0, in, wrows, uint64_t(in) * 2, 64, 128, true));
        if (gateup) G_TRY(g_map(&a.tm_p1, true, p.p1, in, wrows, uint64_t(in) * 2, 64, 128, true));
    } else {
        G_TRY(g_map(&a.tm_p0, false, p.p0, in / 2, wrows, uint64_t(in) / 2, 128, 128, true));
        if (gateup) G_TRY(g_map(&a.tm_p1, false, p.p1, in / 2, wrows, uint64_t(in) / 2, 128, 128, true));
    }
    if (nv) {
        G_TRY(g_map(&a.tm_s0, false, p.s0, in / 16, wrows, uint64_t(in) / 16, 16, 128, false));
        if (gateup) G_TRY(g_map(&a.tm_s1, false, p.s1, in / 16, wrows, uint64_t(in) / 16, 16, 128, false));
    }
    // a tile holds at most min(rows, 128) token rows: only the box heights up to that are encoded
    const int nb_maps = std::min(G_NB_MAPS, (std::min(rows, 128) + 15) / 16);
    if (i8) {
        // three digit rows per activation row, 16 rows and 128 bytes of K per box
        G_TRY(g_map(&a.tm_b[0], false, bsrc, in, uint64_t(rows) * 3, uint64_t(in), 128, 16, true));
    } else if (a4) {
        const uint8_t* codes = static_cast<const uint8_t*>(bsrc);
        for (int i = 0; i < nb_maps; i++) {
            G_TRY(g_map(&a.tm_b[i], false, codes, in / 2, uint64_t(rows), uint64_t(in) / 2, 128, uint32_t(16 * (i + 1)),
                        true));
            G_TRY(g_map(&a.tm_bs[i], false, codes + a4_sc_off, in / 16, uint64_t(rows), uint64_t(in) / 16, 16,
                        uint32_t(16 * (i + 1)), false));
        }
    } else {
        for (int i = 0; i < nb_maps; i++)
            G_TRY(g_map(&a.tm_b[i], true, bsrc, in, uint64_t(rows), uint64_t(in) * 2, 64, uint32_t(16 * (i + 1)), true));
    }
    a.sc0 = reinterpret_cast<const uint8_t*>(p.s0);
    a.sc1 = reinterpret_cast<const uint8_t*>(p.s1);
    a.g0 = p.g0;
    a.g1 = p.g1;
    a.offsets = p.offsets;
    a.row_slot = p.row_slot;
    a.topk_w = p.topk_w;
    a.act_scale = ascale;
    a.out = p.out;
    a.status = p.status;
    a.E = E;
    a.out_dim = out;
    a.in_dim = in;
    a.ksplit = ksplit;
    a.partial = buf.partial;
    a.rows = rows;
    a.zsum = buf.zbuf;
    a.sched = buf.sched;
    a.early = prep_launched ? 1 : 0;
    // wide gate/up tiles (128 token rows) once the experts average more than 64 rows; narrow ones
    // (16) when no expert can hold more than 16 rows (BF16 and the NVFP4 16-bit path)
    const bool wide = gateup && ksplit == 1 && rows > 64 * E;
    const bool narrow = !wide && (p.fmt == MOE_FMT_BF16 || (nv && !a4)) && buf.max_expert_rows > 0 &&
                        buf.max_expert_rows <= 16;
    const int mc = buf.max_ctas;
    const bool pdl = !buf.no_pdl;
    // split-K tiles finish in the GEMM when their counters fit the workspace's control block
    const int nmax = narrow ? 16 : (gateup ? 64 : 128);
    const int ntile_max = (rows + nmax - 1) / nmax;
    if (ksplit > 1 && ksplit <= G_KSPLIT_MAX && buf.tile_cnt && 4 * (out / G_BM) * ntile_max <= kTileCounters)
        a.tile_cnt = buf.tile_cnt;
    if (i8) return gateup ? g_launch<FMT_INT4_I8, true>(a, s, mc, pdl) : g_launch<FMT_INT4_I8, false>(a, s, mc, pdl);
    if (i4) return gateup ? (wide ? g_launch<MOE_FMT_INT4_G128, true, 1>(a, s, mc, pdl) : g_launch<MOE_FMT_INT4_G128, true>(a, s, mc, pdl))
                          : g_launch<MOE_FMT_INT4_G128, false>(a, s, mc, pdl);
    if (a4) return gateup ? (wide ? g_launch<FMT_NVFP4_A4, true, 1>(a, s, mc, pdl) : g_launch<FMT_NVFP4_A4, true>(a, s, mc, pdl))
                          : g_launch<FMT_NVFP4_A4, false>(a, s, mc, pdl);
    if (nv) {
        if (narrow) return gateup ? g_launch<MOE_FMT_NVFP4, true, 2>(a, s, mc, pdl) : g_launch<MOE_FMT_NVFP4, false, 2>(a, s, mc, pdl);
        return gateup ? (wide ? g_launch<MOE_FMT_NVFP4, true, 1>(a, s, mc, pdl) : g_launch<MOE_FMT_NVFP4, true>(a, s, mc, pdl))
                      : g_launch<MOE_FMT_NVFP4, false>(a, s, mc, pdl);
    }
    const int rc = narrow ? (gateup ? g_launch<MOE_FMT_BF16, true, 2>(a, s, mc, pdl) : g_launch<MOE_FMT_BF16, false, 2>(a, s, mc, pdl))
                          : gateup ? (wide ? g_launch<MOE_FMT_BF16, true, 1>(a, s, mc, pdl) : g_launch<MOE_FMT_BF16, true>(a, s, mc, pdl))
                                   : g_launch<MOE_FMT_BF16, false>(a, s, mc, pdl);
    if (rc != MOE_OK) return rc;
    if (ksplit > 1 && !a.tile_cnt) {
        const size_t n4 = size_t(rows) * out / 4;
        const int blocks = int(std::min<size_t>((n4 + 255) / 256, 148 * 8));
        if (launch_pdl(g_splitk_finish, dim3(blocks), dim3(256), 0, s, static_cast<const float*>(buf.partial), ksplit,
                       gateup ? 2 : 1, rows, out, p.topk_w, p.row_slot, p.out) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

}  // namespace moe
