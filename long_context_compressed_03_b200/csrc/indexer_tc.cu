// indexer_tc.cu -- tensor-core Lightning-Indexer scores fused with an exact
// per-query top-k (prefill: 128 consecutive queries of one sequence per CTA).
//
// score[t, s] = ks_s * sum_h w_{t,h} qs_{t,h} * ReLU(q_{t,h} . k_s)   for s < V(t)
// (w: gate weights of any sign, 1 when none are given)
// idx[t, :]   = the topk largest scores, equal scores lowest index first
// ("百万上下文从「奢侈品」变「日用品」…" §3.2 indexer + top-k, §8.2 streaming
//  selection without materialising the scores; "DS-V4 分析&学习" §4 low-
//  precision indexer QK.)  fp8: q and k are E4M3 codes with per-row scales
// qs, ks (the bf16 queries are quantised here, in fp32, exactly as the
// compressor quantises a row); bf16: qs = ks = 1.
//
// Scores: for every chunk of 64 entries the MMA warp issues one tcgen05 MMA
// per indexer head and K step (M = 128 queries, N = 64 entries, K = 64) into
// one of two TMEM buffers (each 4 heads x 64 columns), so the tensor core
// fills one while the epilogue works on the other.  The four epilogue
// warpgroups share a chunk, each taking 16 of its entries; each thread owns
// one query row and folds the heads of its row's scores on packed fp32x2
// arithmetic, with the TMEM loads of the next four columns in flight while
// it works.  Chunks are visited from the middle of the visible entries on.
//
// Selection.  Every (row, entry) has the unique 48-bit key
//   K = (32-bit order-preserving image u of the score) << 16 | (65535 - s),
// which orders like (score desc, index asc) -- the top-k tie rule (u: the
// fp32 bit pattern of a non-negative score, score_key() with gate weights).
// The scores are computed twice on the tensor cores, never stored:
//   pass 1 (window): the first chunk is a probe; the row's probe maximum
//     M (over the four groups' slices, after a barrier of the epilogue
//     warps) anchors a window of 256 bins of 1/64 octave (u >> 17) whose top
//     lies one octave above M.  The pass counts every score into its window
//     bin (scores above the window share one bin; scores below are not
//     counted), so the bin holding the k-th largest key -- and how many keys
//     lie above it -- are exact after one pass;
//   pass 2 (emit): every key above that bin goes to the output row, the
//     keys of the bin itself (at most kCap) to a list, of which the row
//     takes as many of the largest as it still needs.
// A row whose k-th key falls outside the window, or whose boundary bin holds
// more than kCap keys, is resolved instead by an MSB-first radix select over
// the remaining key bits (8-bit digits, one recomputing pass each) before
// the emit pass.  Each selected row is finally written in ascending entry
// order through a bitmap (a deterministic order).  The score matrix never
// leaves the SM.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace csa {
namespace {

using namespace tc;

constexpr int kRows = 128;      // queries per CTA = MMA M
constexpr int kN = 64;          // entries per chunk = MMA N
constexpr int kSlice = kN / 4;  // entries of a chunk that one epilogue group works on
constexpr int kBufs = 2;        // TMEM buffers of kHeads x kN columns (double-buffered)
constexpr int kGroups = 4;      // epilogue warpgroups (one TMEM buffer each)
constexpr int kHeads = 4;       // indexer heads held in TMEM
constexpr int kDim = 64;        // indexer head dim = MMA K
constexpr int kEpiWarps = 4 * kGroups;
constexpr int kThreads = (2 + kEpiWarps) * 32;   // warp 0 TMA, warp 1 MMA, warps 2-17 epilogue
constexpr int kCap = 64;        // boundary keys listed per row
#ifndef CSA_IDX_PART
#define CSA_IDX_PART 4
#endif
constexpr int kPart = CSA_IDX_PART;   // score columns per TMEM load (per head)
constexpr int kWinShift = 17;   // window bin of a score: u >> 17 (1/64 octave)
constexpr int kWinBins = 256;   // window bins (+ bin 0: every score above the window)
constexpr int kWinAbove = 64;   // the window's top bin lies one octave above the probe maximum
constexpr int kHistWords = (kWinBins + 1) * kRows;
static_assert(kRows * kCap * 8 <= kHistWords * 4, "boundary lists alias the histogram");
// after the boundary lists: bitmaps of V <= 65536 bits for at least 8 warps
constexpr int kBitmapWords = (kHistWords * 4 - kRows * kCap * 8) / 4;
static_assert(kBitmapWords >= 8 * 2048, "bitmaps of eight warps fit beside the lists");

enum PassKind { kWindow = 0, kDigit = 1, kEmit32 = 2, kEmit64 = 3 };

template <bool FP8>
struct Cfg {
    static constexpr int kElem = FP8 ? 1 : 2;
    static constexpr int kRowBytes = kDim * kElem;                  // 64 / 128
    static constexpr int kATile = kRows * kRowBytes;                // per head
    static constexpr int kBTile = kN * kRowBytes;                   // per chunk
    // keys are re-read from L2 on every pass: 32 KB (fp8) / 16 KB (bf16) of
    // chunk loads in flight
    static constexpr int kStages = FP8 ? 8 : 2;
    static constexpr int kKSteps = FP8 ? 2 : 4;                     // K=32 (fp8) / 16 (bf16)
    // the window histogram; in the emit pass the boundary lists and, after
    // it, the lists and one bitmap per rewriting warp
    static constexpr int kHist = kHistWords * 4;
};

struct IdxParams {
    const void* qI;            // [B, n, H_I, 64] bf16 or e4m3 codes
    const float* qI_scale;     // e4m3 queries given as codes: [B, n, H_I]
    const float* kI_scale;     // e4m3 keys: [B, N_cap]
    const float* qw;           // gate weights [B, n, H_I] (GATED kernels only)
    int q_mode;                // 0 bf16 (bf16 keys), 1 bf16 quantised here, 2 e4m3 codes,
                               // 3 bf16 Hadamard-rotated, then quantised here
    float hnorm;               // q_mode 3: fp32(1/sqrt(64))
    int B, n, H_I, N_cap, m, topk;
    int pos0;                  // position of query row 0 (a context-parallel shard)
    const int* n_entries;
    int* idx_out;
    uint32_t* err;
    uint64_t wait_ns;          // time limit of each wait of the work
    int stall;                 // test hook: one thread waits on stall_bar first
    VarlenMap vl;              // packed sequences (vl.S > 0): grid.y = sequence
};

struct __align__(8) Ctrl {
    uint64_t full[32];
    uint64_t freeb[32];
    uint64_t acc_full[kBufs];
    uint64_t acc_free[kBufs];
    uint64_t fin;
    uint64_t stall_bar;          // test hook: a barrier nothing completes
    uint32_t tmem_base;
    int abort;
    int kind;                  // the pass about to run
};

// Per-row selection state (shared by the four epilogue groups).
struct RowState {
    uint64_t prefix[kRows];    // key bits above `sh` already decided
    int sh[kRows];             // key bits below the prefix (48: nothing decided)
    int rank[kRows];           // keys still needed from the prefix's bin
    int ready[kRows];          // the next emit pass resolves the row
    int V[kRows];              // visible entries (0 for rows beyond n)
    int emitted[kRows];        // output slots used
    int listed[kRows];         // boundary keys collected
    int T1[kRows];             // window top bin + 1
    uint32_t probe[kGroups][kRows];
    float qs[kRows][kHeads];   // per-head query scales (times the gate weight)
};

template <bool FP8>
constexpr size_t smem_bytes() {
    using C = Cfg<FP8>;
    return 1024 /*alignment slack*/ + (size_t)kHeads * C::kATile + (size_t)C::kStages * C::kBTile +
           C::kHist + (size_t)kEpiWarps * 2 * kSlice * sizeof(float) + sizeof(RowState) + sizeof(Ctrl);
}
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "exceeds the shared-memory limit");

__device__ __forceinline__ int shift_ok32(int sh) { return sh >= 16 && sh <= 47; }

// No-swizzle K-major layout for a [128 x kRowBytes] operand written by threads:
// 8-row x 16-byte core matrices, LBO = 128 B between core matrices along K,
// SBO = (kRowBytes/16) * 128 B between 8-row groups.
template <int kRowBytes>
__device__ __forceinline__ uint32_t a_offset(int r, int chunk16) {
    return (uint32_t)((r >> 3) * (kRowBytes / 16) * 128 + chunk16 * 128 + (r & 7) * 16);
}
__device__ __forceinline__ uint64_t desc_noswizzle(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    return d;   // layout type 0: no swizzle
}
__device__ __forceinline__ uint64_t desc_sw(uint32_t saddr, uint32_t sbo, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)layout << 61;
    return d;
}

// ------------------------------------------------------------------ packed fp32x2
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// (x + |x|, y + |y|) = 2 (ReLU x, ReLU y), exactly (+0 for x <= 0)
__device__ __forceinline__ uint64_t relu2x(float x, float y) {
    return f2_pack(x + fabsf(x), y + fabsf(y));
}

// Four heads x 8 columns (head h at column offset h*kN) with one wait.
__device__ __forceinline__ void tmem_ld8x4(uint32_t taddr, float (&v)[kHeads][8]) {
    uint32_t* r = reinterpret_cast<uint32_t*>(&v[0][0]);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%32];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%8, %9, %10, %11, %12, %13, %14, %15}, [%33];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%16, %17, %18, %19, %20, %21, %22, %23}, [%34];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%24, %25, %26, %27, %28, %29, %30, %31}, [%35];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr), "r"(taddr + kN), "r"(taddr + 2 * kN), "r"(taddr + 3 * kN)
        : "memory");
}
__device__ __forceinline__ void tmem_ldx4(uint32_t taddr, float (&v)[kHeads][8]) { tmem_ld8x4(taddr, v); }
__device__ __forceinline__ void tmem_ldx4(uint32_t taddr, float (&v)[kHeads][4]);   // defined below

// Software-pipelined TMEM loads of one part (four heads x W columns).
// tmem_wait_ld_x4 waits for the part in `cur` (all earlier TMEM loads of this
// thread) and issues the load of the next part into `nxt` in the same
// statement: `cur` is tied through it, so nothing reads its registers before
// the wait, and `nxt` is only read after the statement that waits for it in
// turn.  tmem_ld_x4_nowait issues a load; tmem_wait_x4 only waits.
__device__ __forceinline__ void tmem_wait_ld_x4(float (&cur)[kHeads][4], uint32_t taddr, float (&nxt)[kHeads][4]) {
    uint32_t* c = reinterpret_cast<uint32_t*>(&cur[0][0]);
    uint32_t* r = reinterpret_cast<uint32_t*>(&nxt[0][0]);
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%16, %17, %18, %19}, [%32];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%20, %21, %22, %23}, [%33];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%24, %25, %26, %27}, [%34];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%28, %29, %30, %31}, [%35];\n\t"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3]), "+r"(c[4]), "+r"(c[5]), "+r"(c[6]), "+r"(c[7]), "+r"(c[8]), "+r"(c[9]), "+r"(c[10]), "+r"(c[11]), "+r"(c[12]), "+r"(c[13]), "+r"(c[14]), "+r"(c[15]), "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr), "r"(taddr + kN), "r"(taddr + 2 * kN), "r"(taddr + 3 * kN)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_x4_nowait(uint32_t taddr, float (&nxt)[kHeads][4]) {
    uint32_t* r = reinterpret_cast<uint32_t*>(&nxt[0][0]);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%16];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4, %5, %6, %7}, [%17];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%8, %9, %10, %11}, [%18];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%12, %13, %14, %15}, [%19];\n\t"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr), "r"(taddr + kN), "r"(taddr + 2 * kN), "r"(taddr + 3 * kN)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_x4(float (&cur)[kHeads][4]) {
    uint32_t* c = reinterpret_cast<uint32_t*>(&cur[0][0]);
    asm volatile("tcgen05.wait::ld.sync.aligned;"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3]), "+r"(c[4]), "+r"(c[5]), "+r"(c[6]), "+r"(c[7]), "+r"(c[8]), "+r"(c[9]), "+r"(c[10]), "+r"(c[11]), "+r"(c[12]), "+r"(c[13]), "+r"(c[14]), "+r"(c[15])
        :
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld_x4(float (&cur)[kHeads][8], uint32_t taddr, float (&nxt)[kHeads][8]) {
    uint32_t* c = reinterpret_cast<uint32_t*>(&cur[0][0]);
    uint32_t* r = reinterpret_cast<uint32_t*>(&nxt[0][0]);
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%32, %33, %34, %35, %36, %37, %38, %39}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%40, %41, %42, %43, %44, %45, %46, %47}, [%65];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%48, %49, %50, %51, %52, %53, %54, %55}, [%66];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%56, %57, %58, %59, %60, %61, %62, %63}, [%67];\n\t"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3]), "+r"(c[4]), "+r"(c[5]), "+r"(c[6]), "+r"(c[7]), "+r"(c[8]), "+r"(c[9]), "+r"(c[10]), "+r"(c[11]), "+r"(c[12]), "+r"(c[13]), "+r"(c[14]), "+r"(c[15]), "+r"(c[16]), "+r"(c[17]), "+r"(c[18]), "+r"(c[19]), "+r"(c[20]), "+r"(c[21]), "+r"(c[22]), "+r"(c[23]), "+r"(c[24]), "+r"(c[25]), "+r"(c[26]), "+r"(c[27]), "+r"(c[28]), "+r"(c[29]), "+r"(c[30]), "+r"(c[31]), "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr), "r"(taddr + kN), "r"(taddr + 2 * kN), "r"(taddr + 3 * kN)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_x4_nowait(uint32_t taddr, float (&nxt)[kHeads][8]) {
    uint32_t* r = reinterpret_cast<uint32_t*>(&nxt[0][0]);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%32];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%8, %9, %10, %11, %12, %13, %14, %15}, [%33];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%16, %17, %18, %19, %20, %21, %22, %23}, [%34];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%24, %25, %26, %27, %28, %29, %30, %31}, [%35];\n\t"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr), "r"(taddr + kN), "r"(taddr + 2 * kN), "r"(taddr + 3 * kN)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_x4(float (&cur)[kHeads][8]) {
    uint32_t* c = reinterpret_cast<uint32_t*>(&cur[0][0]);
    asm volatile("tcgen05.wait::ld.sync.aligned;"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3]), "+r"(c[4]), "+r"(c[5]), "+r"(c[6]), "+r"(c[7]), "+r"(c[8]), "+r"(c[9]), "+r"(c[10]), "+r"(c[11]), "+r"(c[12]), "+r"(c[13]), "+r"(c[14]), "+r"(c[15]), "+r"(c[16]), "+r"(c[17]), "+r"(c[18]), "+r"(c[19]), "+r"(c[20]), "+r"(c[21]), "+r"(c[22]), "+r"(c[23]), "+r"(c[24]), "+r"(c[25]), "+r"(c[26]), "+r"(c[27]), "+r"(c[28]), "+r"(c[29]), "+r"(c[30]), "+r"(c[31])
        :
        : "memory");
}

__device__ __forceinline__ void tmem_ldx4(uint32_t taddr, float (&v)[kHeads][4]) {
    tmem_ld_x4_nowait(taddr, v);
    tmem_wait_x4(v);
}

// Per-thread view of its row for one pass.
struct RowCtx {
    int V;
    int T1;                    // window: top bin + 1
    int sh, w;                 // digit pass: bits below the prefix, digit width
    uint32_t wmask;
    uint64_t prefix;
    uint32_t p32;              // emit with sh in [16, 47]: the prefix as a 32-bit value
    int sh32;                  // sh - 16
    uint32_t hrow;             // shared address of hist + row: bin j at hrow + j * kRows * 4
    int* orow;
    uint32_t list;             // shared address of the row's boundary list (u64 keys)
    uint32_t emitted;          // shared addresses of the row's counters
    uint32_t listed;
    int topk;
    uint64_t c2[kHeads];       // (c_h, c_h): half the head's query scale (times its gate weight)
};

// Shared-memory atomics on 32-bit shared addresses.  The counting passes
// take the predicated form: one instruction per score, no branch.
__device__ __forceinline__ void red_add_shared_if(uint32_t addr, bool pred) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\t@p red.shared.add.u32 [%0], 1;\n\t}"
                 ::"r"(addr), "r"((uint32_t)pred) : "memory");
}
__device__ __forceinline__ int atom_add_shared(uint32_t addr, int v) {
    int old;
    asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}

// A key in the boundary bin goes to the row's list (rare: a few dozen per row).
__device__ __forceinline__ void list_one(uint64_t key, const RowCtx& rc) {
    const int pos = atom_add_shared(rc.listed, 1);
    if (pos < kCap) asm volatile("st.shared.u64 [%0], %1;" ::"r"(rc.list + 8u * pos), "l"(key) : "memory");
}

// The certain keys of a slice (bit b: entry e0 + b) go to the output row:
// one shared atomic per row and slice claims their slots.
__device__ __forceinline__ void emit_slice(uint32_t mask, int e0, const RowCtx& rc) {
    if (!mask) return;
    int pos = atom_add_shared(rc.emitted, __popc(mask));
    while (mask) {
        const int b = __ffs(mask) - 1;
        mask &= mask - 1u;
        if (pos < rc.topk) rc.orow[pos] = e0 + b;
        ++pos;
    }
}

enum { kProbe = 4 };

// One score of this thread's row, by pass kind.
template <int MODE, bool GATED>
__device__ __forceinline__ void take(float sc, int s, const RowCtx& rc, uint32_t& mx) {
    const uint32_t u = GATED ? score_key(sc) : __float_as_uint(sc);
    if constexpr (MODE == kProbe) {
        mx = max(mx, u);
    } else if constexpr (MODE == kWindow) {
        const int jj = max(rc.T1 - (int)(u >> kWinShift), 0);
        red_add_shared_if(rc.hrow + (uint32_t)jj * (kRows * 4), jj <= kWinBins);
    } else if constexpr (MODE == kDigit) {
        const uint64_t key = ((uint64_t)u << 16) | (uint64_t)(65535 - s);
        red_add_shared_if(rc.hrow + (uint32_t)((key >> (rc.sh - rc.w)) & rc.wmask) * (kRows * 4),
                          (key >> rc.sh) == rc.prefix);
    } else if constexpr (MODE == kEmit32) {
        // mx collects the slice's certain keys (bit s mod kSlice)
        const uint32_t kp = u >> rc.sh32;
        if (kp > rc.p32) mx |= 1u << (s & (kSlice - 1));
        else if (kp == rc.p32) list_one(((uint64_t)u << 16) | (uint64_t)(65535 - s), rc);
    } else {
        const uint64_t key = ((uint64_t)u << 16) | (uint64_t)(65535 - s);
        const uint64_t kp = key >> rc.sh;
        if (kp > rc.prefix) mx |= 1u << (s & (kSlice - 1));
        else if (kp == rc.prefix) list_one(key, rc);
    }
}

// Scores e, e+1 of a kPart-column part: sum_h c_h (a_h + |a_h|), times the key
// scales (fp8), on packed fp32x2 arithmetic.
template <bool FP8>
__device__ __forceinline__ uint64_t fold2(const float (&a)[kHeads][kPart], int e, const uint64_t (&c2)[kHeads],
                                          float k0, float k1) {
    uint64_t acc = f2_mul(relu2x(a[0][e], a[0][e + 1]), c2[0]);
#pragma unroll
    for (int h = 1; h < kHeads; ++h) acc = f2_fma(relu2x(a[h][e], a[h][e + 1]), c2[h], acc);
    if (FP8) acc = f2_mul(acc, f2_pack(k0, k1));
    return acc;
}

// The kPart scores of one part (columns s0 .. s0+kPart-1 of this thread's
// row), already in registers.  ksb: the chunk's key scales in the warp's
// shared-memory slot (fp8).
template <bool FP8, bool GATED, int MODE>
__device__ __forceinline__ void part_work(const float (&a)[kHeads][kPart], const float* ksb, int s0,
                                          const RowCtx& rc, uint32_t& mx) {
    if (s0 + kPart <= rc.V) {
#pragma unroll
        for (int e = 0; e < kPart; e += 4) {
            float4 k4 = make_float4(1.f, 1.f, 1.f, 1.f);
            if (FP8) k4 = *reinterpret_cast<const float4*>(ksb + e);
            const uint64_t v0 = fold2<FP8>(a, e, rc.c2, k4.x, k4.y);
            const uint64_t v1 = fold2<FP8>(a, e + 2, rc.c2, k4.z, k4.w);
            if constexpr (MODE == kEmit32 || MODE == kEmit64) {
                // the four keys' certain bits into mx, the rare boundary keys
                // after them: one branch per four scores
                const float sc[4] = {f2_lo(v0), f2_hi(v0), f2_lo(v1), f2_hi(v1)};
                uint32_t eq = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t u = GATED ? score_key(sc[i]) : __float_as_uint(sc[i]);
                    const int si = s0 + e + i;
                    bool gt, same;
                    if constexpr (MODE == kEmit32) {
                        const uint32_t kp = u >> rc.sh32;
                        gt = kp > rc.p32;
                        same = kp == rc.p32;
                    } else {
                        const uint64_t kp = (((uint64_t)u << 16) | (uint64_t)(65535 - si)) >> rc.sh;
                        gt = kp > rc.prefix;
                        same = kp == rc.prefix;
                    }
                    mx |= (gt ? 1u : 0u) << (si & (kSlice - 1));
                    eq |= (same ? 1u : 0u) << i;
                }
                if (eq) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if ((eq >> i) & 1u) {
                            const uint32_t u = GATED ? score_key(sc[i]) : __float_as_uint(sc[i]);
                            list_one(((uint64_t)u << 16) | (uint64_t)(65535 - (s0 + e + i)), rc);
                        }
                }
            } else {
                take<MODE, GATED>(f2_lo(v0), s0 + e, rc, mx);
                take<MODE, GATED>(f2_hi(v0), s0 + e + 1, rc, mx);
                take<MODE, GATED>(f2_lo(v1), s0 + e + 2, rc, mx);
                take<MODE, GATED>(f2_hi(v1), s0 + e + 3, rc, mx);
            }
        }
    } else {
#pragma unroll
        for (int e = 0; e < kPart; e += 2) {
            const float k0 = FP8 ? ksb[e] : 1.f, k1 = FP8 ? ksb[e + 1] : 1.f;
            const uint64_t v = fold2<FP8>(a, e, rc.c2, k0, k1);
            if (s0 + e < rc.V) take<MODE, GATED>(f2_lo(v), s0 + e, rc, mx);
            if (s0 + e + 1 < rc.V) take<MODE, GATED>(f2_hi(v), s0 + e + 1, rc, mx);
        }
    }
}

// Chunk visited at position i of a pass over n chunks: from the middle on,
// wrapping around.
__device__ __forceinline__ int chunk_pos(int i, int n) {
    const int c = i + (n >> 1);
    return c >= n ? c - n : c;
}

// The probe: the largest key of this thread's row in the group's slice of
// one chunk (e0: its first entry; loads wait in place; once per CTA).
template <bool FP8, bool GATED>
__device__ __forceinline__ uint32_t slice_probe(uint32_t taddr, const float* ksb, int e0, bool active,
                                                const RowCtx& rc) {
    uint32_t mx = 0;
#pragma unroll 1
    for (int part = 0; part < kSlice / kPart; ++part) {
        float a[kHeads][kPart];
        tmem_ldx4(taddr + part * kPart, a);
        if (active) part_work<FP8, GATED, kProbe>(a, ksb + part * kPart, e0 + part * kPart, rc, mx);
    }
    return mx;
}

// One pass of an epilogue group over every chunk (its slice of columns of
// each), with the TMEM loads software-pipelined: the load of the next part
// (of this slice, or the first part of the next chunk's slice, which the
// tensor core has written into the other buffer) is in flight while a part
// is worked on.  The warp releases a buffer as soon as its slice is in
// registers.  Returns false when a wait gave up (abort).
template <bool FP8, bool GATED, int MODE>
__device__ __forceinline__ bool group_pass(Ctrl* ctl, uint32_t tbase, float* ksb2, int grp, int nchunks,
                                           bool active, const RowCtx& rc, int (&cons)[kBufs], float& ksv,
                                           const float* ksc, int Vmax, volatile int* abort, uint32_t* err,
                                           uint64_t wait_ns, bool first_waited) {
    constexpr int kParts = kSlice / kPart;
    static_assert(kParts % 2 == 0, "parts alternate between two register sets");
    const int lane = threadIdx.x & 31;
    auto slice0 = [&](int i) -> int { return chunk_pos(i, nchunks) * kN + grp * kSlice; };
    auto scale_at = [&](int i) -> float {
        if (!FP8 || i >= nchunks) return 0.0f;
        const int e = slice0(i) + lane;
        return (lane < kSlice && e < Vmax) ? __ldg(ksc + e) : 0.0f;
    };
    if (nchunks <= 0) return true;
    int i = 0, buf = 0;
    const uint32_t col0 = tbase + grp * kSlice;
    if (!first_waited) {
        if (!__all_sync(0xffffffffu, mbar_wait(&ctl->acc_full[0], cons[0] & 1, abort, err, wait_ns))) return false;
        tc_fence_after();
        if (FP8) {
            __syncwarp();
            if (lane < kSlice) ksb2[lane] = ksv;
            __syncwarp();
        }
    }
    float ksv_next = scale_at(1);
    float A[kHeads][kPart], B[kHeads][kPart];
    uint32_t mx = 0;
    tmem_ld_x4_nowait(col0, A);
    while (true) {
        const int e0 = slice0(i);
        const uint32_t taddr = col0 + buf * (kHeads * kN);
        const int bufn = buf ^ 1;
        bool more = i + 1 < nchunks;
#pragma unroll
        for (int q = 0; q < kParts; q += 2) {
            tmem_wait_ld_x4(A, taddr + (q + 1) * kPart, B);            // part q ready, q+1 in flight
            if (active) part_work<FP8, GATED, MODE>(A, ksb2 + buf * kSlice + q * kPart, e0 + q * kPart, rc, mx);
            if (q + 2 < kParts) {
                tmem_wait_ld_x4(B, taddr + (q + 2) * kPart, A);        // part q+1 ready, q+2 in flight
            } else {
                if (more) {
                    more = __all_sync(0xffffffffu, mbar_wait(&ctl->acc_full[bufn], cons[bufn] & 1, abort, err, wait_ns));
                    if (more) tc_fence_after();
                }
                if (more)
                    tmem_wait_ld_x4(B, col0 + bufn * (kHeads * kN), A);   // next chunk in flight
                else
                    tmem_wait_x4(B);
                // this slice is in registers: the warp's share of the buffer is free
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->acc_free[buf]);
                ++cons[buf];
            }
            if (active)
                part_work<FP8, GATED, MODE>(B, ksb2 + buf * kSlice + (q + 1) * kPart, e0 + (q + 1) * kPart, rc, mx);
        }
        if constexpr (MODE == kEmit32 || MODE == kEmit64) {
            if (active) emit_slice(mx, e0, rc);
            mx = 0;
        }
        if (!more) break;
        // the next chunk's key scales into the warp's other slot
        if (FP8) {
            __syncwarp();
            if (lane < kSlice) ksb2[bufn * kSlice + lane] = ksv_next;
            __syncwarp();
        }
        ++i;
        buf = bufn;
        ksv_next = scale_at(i + 1);
    }
    return !*abort;
}

// 18 warps sit on the SM's four 16,384-register partitions as 5 + 5 + 4 + 4,
// so a thread may hold at most 96 registers.
template <bool FP8, bool GATED>
__global__ void __maxnreg__(96)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tm_k, IdxParams p) {
    using C = Cfg<FP8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;                                       // [kHeads][kATile]
    uint8_t* sB = sA + kHeads * C::kATile;                    // [kStages][kBTile]
    uint32_t* hist = reinterpret_cast<uint32_t*>(sB + C::kStages * C::kBTile);   // [257][128]
    uint64_t* list = reinterpret_cast<uint64_t*>(hist);      // [128][kCap] (aliases hist)
    float* ksbuf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(hist) + C::kHist);   // [16][2][kN]
    RowState* rs = reinterpret_cast<RowState*>(ksbuf + kEpiWarps * 2 * kSlice);
    Ctrl* ctl = reinterpret_cast<Ctrl*>(rs + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's 128 queries: element (or packed sequence) b, rows t0 .. of
    // its slen; its rows start at token tok0 and entry ent0; row t sits at
    // position pos0 + t.  Heavy tiles (late queries see more entries) first.
    int b, t0, slen, ne;
    size_t tok0, ent0;
    if (p.vl.S) {
        b = blockIdx.y;
        tok0 = (size_t)p.vl.tok[b];
        ent0 = (size_t)p.vl.ent[b];
        slen = p.vl.tok[b + 1] - p.vl.tok[b];
        ne = slen / p.m;
        t0 = (gridDim.x - 1 - blockIdx.x) * kRows;
        if (t0 >= slen) return;    // a shorter sequence: nothing set up yet, the whole CTA leaves
    } else {
        const int tiles_per_seq = (p.n + kRows - 1) / kRows;
        const int tile = gridDim.x - 1 - blockIdx.x;
        b = tile / tiles_per_seq;
        t0 = (tile - b * tiles_per_seq) * kRows;
        slen = p.n;
        tok0 = (size_t)b * p.n;
        ent0 = (size_t)b * p.N_cap;
        ne = clampi(p.n_entries ? p.n_entries[b] : p.N_cap, 0, p.N_cap);
    }
    const int t_last = min(t0 + kRows - 1, slen - 1);
    const int Vmax = min((p.pos0 + t_last + 1) / p.m, ne);
    const int nchunks = (Vmax + kN - 1) / kN;
    // chunk visited at position i: from the middle of the visible entries on,
    // so that the first chunk (the window's probe) is one no row is short of
    auto chunk_at = [&](int i) -> int { return chunk_pos(i, nchunks); };
    volatile int* abort = &ctl->abort;

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->freeb[s], 1);
        }
        for (int g = 0; g < kBufs; ++g) {
            mbar_init(&ctl->acc_full[g], 1);
            mbar_init(&ctl->acc_free[g], kEpiWarps);   // one arrival per epilogue warp
        }
        mbar_init(&ctl->fin, 1);
        mbar_init(&ctl->stall_bar, 1);
        ctl->abort = (*reinterpret_cast<volatile uint32_t*>(p.err) != 0u) ? 1 : 0;
        ctl->kind = kWindow;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, 512);
        tmem_relinquish();
    }
    for (int r = threadIdx.x; r < kRows; r += kThreads) {
        const int t = t0 + r;
        const int V = (t < slen) ? min((p.pos0 + t + 1) / p.m, ne) : 0;
        rs->V[r] = V;
        rs->prefix[r] = 0;
        rs->sh[r] = 48;
        rs->rank[r] = p.topk;
        rs->ready[r] = (V <= p.topk) ? 1 : 0;   // rows with V <= k take every visible entry
        rs->emitted[r] = 0;
        rs->listed[r] = 0;
        rs->T1[r] = 0;
    }
    // the query operand: one warp per (row, head) pair
    // (each lane holds elements 2*lane, 2*lane+1 of the row; four pairs per
    // warp have their loads in flight together)
    constexpr int kWarpsAll = kThreads / 32;
    for (int pair0 = warp; pair0 < kRows * kHeads; pair0 += 4 * kWarpsAll) {
        uint32_t raw[4];
        float qsr[4], qwr[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int pair = pair0 + j * kWarpsAll;
            raw[j] = 0u;
            qsr[j] = 1.0f;
            qwr[j] = 1.0f;
            if (pair < kRows * kHeads) {
                const int r = pair >> 2, h = pair & 3;
                const int t = min(t0 + r, slen - 1);
                const size_t qrow = (tok0 + t) * p.H_I + h;
                if (h < p.H_I) {
                    if (p.q_mode == 2) {
                        raw[j] = reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(p.qI) + qrow * kDim)[lane];
                        qsr[j] = p.qI_scale[qrow];
                    } else {
                        raw[j] = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(p.qI) + qrow * kDim)[lane];
                    }
                    if (GATED) qwr[j] = p.qw[qrow];
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int pair = pair0 + j * kWarpsAll;
            if (pair >= kRows * kHeads) break;      // warp-uniform
            const int r = pair >> 2, h = pair & 3;
            float qs = qsr[j];
            uint32_t packed;              // two output elements (fp8: 2 bytes; bf16: 4 bytes)
            if (h < p.H_I) {
                if (p.q_mode == 2) {
                    packed = raw[j];
                } else {
                    float v0 = __uint_as_float(raw[j] << 16);              // bf16 -> fp32, exact
                    float v1 = __uint_as_float(raw[j] & 0xffff0000u);
                    if (p.q_mode == 3) {
                        // Walsh-Hadamard butterflies in stride order 1, 2, ..., 32:
                        // stride 1 pairs this lane's two elements, stride 2s pairs
                        // lane with lane ^ s (the lower lane holds the left operand).
                        const float a0 = v0;
                        v0 = a0 + v1;
                        v1 = a0 - v1;
#pragma unroll
                        for (int sl = 1; sl < 32; sl <<= 1) {
                            const float p0 = __shfl_xor_sync(0xffffffffu, v0, sl);
                            const float p1 = __shfl_xor_sync(0xffffffffu, v1, sl);
                            const bool hi = (lane & sl) != 0;
                            v0 = hi ? p0 - v0 : v0 + p0;
                            v1 = hi ? p1 - v1 : v1 + p1;
                        }
                        v0 = v0 * p.hnorm;
                        v1 = v1 * p.hnorm;
                    }
                    if (p.q_mode == 1 || p.q_mode == 3) {
                        float amax = fmaxf(fabsf(v0), fabsf(v1));
                        for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
                        qs = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                        packed = (uint32_t)e4m3_code(__fdiv_rn(v0, qs)) | ((uint32_t)e4m3_code(__fdiv_rn(v1, qs)) << 8);
                    } else {
                        packed = raw[j];          // bf16 queries for bf16 keys, as given
                    }
                }
            } else {
                packed = 0u;              // absent head: zero queries score zero
            }
            uint8_t* at = sA + h * C::kATile;
            const int byte = 2 * lane * C::kElem;                    // byte offset of element 2*lane
            const uint32_t off = a_offset<C::kRowBytes>(r, byte >> 4) + (byte & 15);
            if (FP8)
                *reinterpret_cast<uint16_t*>(at + off) = (uint16_t)packed;
            else
                *reinterpret_cast<uint32_t*>(at + off) = packed;
            if (GATED && h < p.H_I) qs *= qwr[j];
            if (lane == 0) rs->qs[r][h] = (h < p.H_I) ? qs : 0.0f;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    // any row that needs selection at all?
    int need = 0;
    for (int r = 0; r < kRows; ++r) need |= (t0 + r < slen && rs->V[r] > p.topk);

    // role counters that persist across passes
    int L = 0;                 // producer / MMA: chunk loads issued
    int use_buf[kBufs] = {0, 0};   // MMA: issues into each TMEM buffer
    int cons[kBufs] = {0, 0};      // epilogue: chunks consumed from each buffer
    const bool is_epi = warp >= 2;
    const int grp = is_epi ? ((warp - 2) >> 2) : 0;      // warps 2-5, 6-9, 10-13, 14-17
    const int r = (warp & 3) * 32 + lane;                    // epilogue row
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;

    for (int pass = 0; need && pass < 9; ++pass) {
        const int kind = ctl->kind;
        const bool emit = kind == kEmit32;
        if (!emit) {
            for (int i = threadIdx.x; i < kHistWords; i += kThreads) hist[i] = 0u;
        }
        __syncthreads();
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                // test hook: a wait that runs out (nothing completes stall_bar)
                if (p.stall && pass == 0) mbar_wait(&ctl->stall_bar, 0, abort, p.err, p.wait_ns);
                for (int i = 0; i < nchunks; ++i, ++L) {
                    const int slot = L % C::kStages, u = L / C::kStages;
                    if (*abort) break;     // nothing is issued once the CTA aborts
                    if (u > 0 && !mbar_wait(&ctl->freeb[slot], (u - 1) & 1, abort, p.err, p.wait_ns)) break;
                    mbar_arrive_expect_tx(&ctl->full[slot], C::kBTile);
                    tma_load_2d(sB + slot * C::kBTile, &tm_k, 0, (int)ent0 + chunk_at(i) * kN, &ctl->full[slot]);
                }
            }
            __syncwarp();
            L = __shfl_sync(0xffffffffu, L, 0);
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                const uint32_t idesc = FP8 ? idesc_e4m3(kRows, kN) : idesc_bf16(kRows, kN, false, false);
                for (int i = 0; i < nchunks; ++i, ++L) {
                    const int slot = L % C::kStages;
                    const int g = i % kBufs;
                    if (!mbar_wait(&ctl->full[slot], (L / C::kStages) & 1, abort, p.err, p.wait_ns)) break;
                    if (use_buf[g] > 0 && !mbar_wait(&ctl->acc_free[g], (use_buf[g] - 1) & 1, abort, p.err, p.wait_ns)) break;
                    tc_fence_after();
                    const uint32_t bsa = smem_u32(sB + slot * C::kBTile);
                    for (int h = 0; h < kHeads; ++h) {
                        const uint32_t asa = smem_u32(sA + h * C::kATile);
                        for (int k = 0; k < C::kKSteps; ++k) {
                            // each K step covers 32 bytes of a row
                            const uint64_t ad = desc_noswizzle(asa + k * 256, 128, (C::kRowBytes / 16) * 128);
                            const uint64_t bd = FP8 ? desc_sw(bsa + k * 32, 512, 4 /*SW64*/)
                                                    : desc_sw(bsa + k * 32, 1024, 2 /*SW128*/);
                            if (FP8)
                                mma_f8_ss(tmem + g * (kHeads * kN) + h * kN, ad, bd, idesc, k > 0);
                            else
                                mma_bf16_ss(tmem + g * (kHeads * kN) + h * kN, ad, bd, idesc, k > 0);
                        }
                    }
                    mma_commit(&ctl->acc_full[g]);
                    mma_commit(&ctl->freeb[slot]);
                    ++use_buf[g];
                }
            }
            __syncwarp();
            L = __shfl_sync(0xffffffffu, L, 0);
            for (int g = 0; g < kBufs; ++g) use_buf[g] = __shfl_sync(0xffffffffu, use_buf[g], 0);
        } else {
            // ------------------------------------------------------------ epilogue
            const int V = rs->V[r];
            const bool sel = t0 + r < slen && V > p.topk;            // the row selects at all
            const bool active = sel && (kind != kDigit || rs->ready[r] == 0);
            RowCtx rc;
            rc.V = V;
            rc.T1 = rs->T1[r];
            rc.sh = rs->sh[r];
            rc.w = min(8, rc.sh);
            rc.wmask = (1u << rc.w) - 1u;
            rc.prefix = rs->prefix[r];
            rc.p32 = (uint32_t)rc.prefix;
            rc.sh32 = rc.sh - 16;
            rc.hrow = smem_u32(hist + r);
            rc.orow = p.idx_out + (tok0 + min(t0 + r, slen - 1)) * p.topk;
            rc.list = smem_u32(list + r * kCap);
            rc.emitted = smem_u32(&rs->emitted[r]);
            rc.listed = smem_u32(&rs->listed[r]);
            rc.topk = p.topk;
#pragma unroll
            for (int h = 0; h < kHeads; ++h) {
                const float c = 0.5f * rs->qs[r][h];   // exact: a power of two
                rc.c2[h] = f2_pack(c, c);
            }
            // emit: the 32-bit comparison serves the warp when every selecting
            // row's prefix lies within the score bits
            int wmode = kind;
            if (emit) wmode = __all_sync(0xffffffffu, !active || shift_ok32(rc.sh)) ? kEmit32 : kEmit64;
            float* ksb2 = ksbuf + (warp - 2) * 2 * kSlice;   // the warp's two key-scale slots
            const float* ksc = FP8 ? p.kI_scale + ent0 : nullptr;
            float ksv = 0.0f;                                // this lane's scale in the first chunk's slice
            if (FP8 && nchunks > 0) {
                const int e = chunk_at(0) * kN + grp * kSlice + lane;
                ksv = (lane < kSlice && e < Vmax) ? __ldg(ksc + e) : 0.0f;
            }
            const uint32_t tbase = tmem + lane_addr;
            bool first_waited = false;
            bool ok = true;
            if (kind == kWindow) {
                // the probe: the first chunk's largest key of the row; the window
                // top follows from the largest of the four groups' probes.  Every
                // epilogue warp joins the barrier once, with or without a chunk.
                uint32_t mx = 0;
                if (nchunks > 0) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&ctl->acc_full[0], cons[0] & 1, abort, p.err, p.wait_ns));
                    if (ok) {
                        tc_fence_after();
                        if (FP8) {
                            __syncwarp();
                            if (lane < kSlice) ksb2[lane] = ksv;
                            __syncwarp();
                        }
                        mx = slice_probe<FP8, GATED>(tbase + grp * kSlice, ksb2, chunk_at(0) * kN + grp * kSlice,
                                                     sel, rc);
                        first_waited = true;
                    }
                }
                rs->probe[grp][r] = mx;
                named_sync(1, kEpiWarps * 32);
                uint32_t M = rs->probe[0][r];
#pragma unroll
                for (int g = 1; g < kGroups; ++g) M = max(M, rs->probe[g][r]);
                rc.T1 = (int)(M >> kWinShift) + kWinAbove + 1;
                if (grp == 0) rs->T1[r] = rc.T1;
            }
            if (ok) {
                switch (wmode) {
                    case kWindow:
                        group_pass<FP8, GATED, kWindow>(ctl, tbase, ksb2, grp, nchunks, active, rc, cons, ksv,
                                                        ksc, Vmax, abort, p.err, p.wait_ns, first_waited);
                        break;
                    case kDigit:
                        group_pass<FP8, GATED, kDigit>(ctl, tbase, ksb2, grp, nchunks, active, rc, cons, ksv,
                                                       ksc, Vmax, abort, p.err, p.wait_ns, first_waited);
                        break;
                    case kEmit32:
                        group_pass<FP8, GATED, kEmit32>(ctl, tbase, ksb2, grp, nchunks, active, rc, cons, ksv,
                                                        ksc, Vmax, abort, p.err, p.wait_ns, first_waited);
                        break;
                    default:
                        group_pass<FP8, GATED, kEmit64>(ctl, tbase, ksb2, grp, nchunks, active, rc, cons, ksv,
                                                        ksc, Vmax, abort, p.err, p.wait_ns, first_waited);
                        break;
                }
            }
        }
        __syncthreads();
        if (*abort) break;
        // ---------------------------------------------------------------- per-row bookkeeping
        if (is_epi && grp == 0) {
            const int V = rs->V[r];
            const bool sel = t0 + r < slen && V > p.topk;
            if (kind == kWindow && sel) {
                // the bin holding the k-th key: bin 0 counts every key above the
                // window, bin j >= 1 the keys whose window prefix is T1 - j
                const int rank = p.topk;
                int cum = (int)hist[r];
                bool found = false;
                if (cum < rank) {
                    for (int j = 1; j <= kWinBins; ++j) {
                        const int cnt = (int)hist[j * kRows + r];
                        if (cum + cnt >= rank) {
                            rs->prefix[r] = (uint64_t)(rs->T1[r] - j);
                            rs->sh[r] = kWinShift + 16;
                            rs->rank[r] = rank - cum;
                            rs->ready[r] = cnt <= kCap ? 1 : 0;
                            found = true;
                            break;
                        }
                        cum += cnt;
                    }
                }
                if (!found) {
                    // the k-th key lies outside the window: radix select from the top bit
                    rs->prefix[r] = 0;
                    rs->sh[r] = 48;
                    rs->rank[r] = rank;
                    rs->ready[r] = 0;
                }
            } else if (kind == kDigit && sel && rs->ready[r] == 0) {
                const int sh = rs->sh[r], w = min(8, sh);
                const int rank = rs->rank[r];
                int cum = 0;
                for (int d = (1 << w) - 1; d >= 0; --d) {
                    const int cnt = (int)hist[d * kRows + r];
                    if (cum + cnt >= rank) {
                        rs->prefix[r] = (rs->prefix[r] << w) | (uint64_t)d;
                        rs->sh[r] = sh - w;
                        rs->rank[r] = rank - cum;
                        rs->ready[r] = (cnt <= kCap || sh - w == 0) ? 1 : 0;
                        break;
                    }
                    cum += cnt;
                }
            }
        }
        __syncthreads();
        if (emit) {
            // the emitted set is exact; its order depends on which group got
            // there first.  Rewrite each selected row in ascending entry order
            // (deterministic and gather-friendly): one warp per row marks the
            // entries in a bitmap over [0, V) in shared memory, then walks it.
            if (is_epi) {
                // one warp per row.  The row's entries are marked in a bitmap
                // over [0, V) in shared memory: the certain keys the pass wrote
                // to the output row, and the `rank` largest keys of the boundary
                // list (a key is taken when fewer than `rank` listed keys exceed
                // it; keys are unique).  The bitmap is then written back as the
                // ascending list of entries: deterministic and gather-friendly.
                const int ew = warp - 2;
                // as many rewriting warps as bitmaps of the CTA's longest row fit
                const int nwv = (Vmax + 31) >> 5;
                const int nrw = min(kEpiWarps, kBitmapWords / max(nwv, 1));
                uint32_t* bm = hist + kRows * kCap * 2 + ew * nwv;
                const int kk = p.topk;
                for (int rr = ew; ew < nrw && rr < kRows; rr += nrw) {
                    if (t0 + rr >= slen) continue;
                    const int V = rs->V[rr];
                    int* orow = p.idx_out + (tok0 + t0 + rr) * kk;
                    if (V <= kk) {
                        // every visible entry, then -1 padding (coalesced)
                        for (int j = lane; j < kk; j += 32) orow[j] = j < V ? j : -1;
                        continue;
                    }
                    const int nw = (V + 31) >> 5;
                    for (int i = lane; i < nw; i += 32) bm[i] = 0u;
                    __syncwarp();
                    const int ne = min(rs->emitted[rr], kk);
                    for (int b0 = 0; b0 < ne; b0 += 32 * 16) {
                        int v[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int i = b0 + j * 32 + lane;
                            v[j] = i < ne ? orow[i] : -1;
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (v[j] >= 0 && v[j] < V) atomicOr(&bm[v[j] >> 5], 1u << (v[j] & 31));
                    }
                    const int nl = min(rs->listed[rr], kCap);
                    const int rank = rs->rank[rr];
                    const uint64_t* lr = list + rr * kCap;
                    for (int i = lane; i < nl; i += 32) {
                        const uint64_t key = lr[i];
                        int above = 0;
                        for (int j = 0; j < nl; ++j) above += lr[j] > key ? 1 : 0;
                        if (above < rank) {
                            const int sidx = 65535 - (int)(key & 0xFFFFu);
                            if (sidx >= 0 && sidx < V) atomicOr(&bm[sidx >> 5], 1u << (sidx & 31));
                        }
                    }
                    __syncwarp();
                    // lane l owns words [l*per, (l+1)*per): one warp scan of the counts
                    const int per = (nw + 31) >> 5;
                    const int w_lo = min(lane * per, nw), w_hi = min(w_lo + per, nw);
                    int cnt = 0;
                    for (int w = w_lo; w < w_hi; ++w) cnt += __popc(bm[w]);
                    int incl = cnt;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const int v = __shfl_up_sync(0xffffffffu, incl, off);
                        if (lane >= off) incl += v;
                    }
                    const int total = __shfl_sync(0xffffffffu, incl, 31);
                    int pos = incl - cnt;
                    for (int w = w_lo; w < w_hi && pos < kk; ++w) {
                        uint32_t word = bm[w];
                        while (word && pos < kk) {
                            const int bit = __ffs(word) - 1;
                            word &= word - 1u;
                            orow[pos++] = (w << 5) + bit;
                        }
                    }
                    for (int j = total + lane; j < kk; j += 32) orow[j] = -1;   // only if counts disagree
                    __syncwarp();
                }
            }
            break;
        }
        // the next pass emits once every selecting row is ready
        if (threadIdx.x == 0) {
            int all_ready = 1;
            for (int i = 0; i < kRows; ++i) all_ready &= rs->ready[i];
            ctl->kind = all_ready ? kEmit32 : kDigit;
        }
        __syncthreads();
    }
    // key loads still in flight after an abort must land before the CTA's
    // shared memory is given up: the last load of each stage is the latest
    // phase of its barrier, so waiting on it covers every earlier one
    if (warp == 0 && lane == 0) {
        volatile int never = 0;
        for (int Lp = max(0, L - C::kStages); Lp < L; ++Lp)
            mbar_wait(&ctl->full[Lp % C::kStages], (Lp / C::kStages) & 1, &never, p.err);
    }
    if (!need) {
        // every row takes all its visible entries (one warp per row, coalesced)
        for (int rr = warp; rr < kRows; rr += kThreads / 32) {
            if (t0 + rr >= slen) continue;
            int* orow = p.idx_out + (tok0 + t0 + rr) * p.topk;
            const int V = rs->V[rr];
            for (int j = lane; j < p.topk; j += 32) orow[j] = j < V ? j : -1;
        }
    }
    // no MMA may be in flight when TMEM is released
    if (warp == 1) {
        if (lane == 0) {
            mma_commit(&ctl->fin);
            volatile int never = 0;
            mbar_wait(&ctl->fin, 0, &never, p.err);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

template <bool FP8, bool GATED>
cudaError_t launch_k(dim3 grid, const CUtensorMap& tm, const IdxParams& p, cudaStream_t s) {
    auto k = indexer_tc_kernel<FP8, GATED>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes<FP8>());
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, smem_bytes<FP8>(), s>>>(tm, p);
    return cudaSuccess;
}

}  // namespace

bool indexer_tc_supported(const IndexerArgs& a) {
    const bool fp8 = (a.kI_dt == DT_E4M3 || a.kI_dt == DT_E4M3H) &&
                     (a.qI_dt == DT_BF16 || a.qI_dt == DT_E4M3);
    const bool bf16 = a.kI_dt == DT_BF16 && a.qI_dt == DT_BF16;
    return (fp8 || bf16) && a.d_I == kDim && a.H_I <= kHeads && a.q_pos == nullptr &&
           a.N_cap <= 65536 && a.n_q >= 1;
}

cudaError_t launch_indexer_tc(const IndexerArgs& a, uint32_t* err, cudaStream_t s) {
    const bool fp8 = a.kI_dt == DT_E4M3 || a.kI_dt == DT_E4M3H;
    auto fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    CUtensorMap tm;
    const int row_bytes = fp8 ? kDim : kDim * 2;
    cuuint64_t dims[2] = {(cuuint64_t)(fp8 ? kDim : kDim), (cuuint64_t)a.B * (a.N_cap > 0 ? a.N_cap : 1)};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)kDim, (cuuint32_t)kN};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&tm, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(a.kI), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    fp8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    IdxParams p;
    p.qI = a.qI;
    p.qI_scale = a.qI_scale;
    p.kI_scale = a.kI_scale;
    p.q_mode = fp8 ? (a.qI_dt == DT_E4M3 ? 2 : (a.kI_dt == DT_E4M3H ? 3 : 1)) : 0;
    p.hnorm = a.hnorm;
    p.B = a.B;
    p.n = a.n_q;
    p.H_I = a.H_I;
    p.N_cap = a.N_cap;
    p.m = a.m;
    p.topk = a.topk;
    p.n_entries = a.n_entries;
    p.idx_out = a.idx_out;
    p.pos0 = a.vl ? 0 : a.pos0;
    p.err = err;
    p.wait_ns = wait_limit_ns();
    p.stall = take_stall();
    p.qw = a.qI_weight;
    const int tiles = (a.n_q + kRows - 1) / kRows;
    dim3 grid((unsigned)(a.B * tiles));
    if (a.vl) {                       // packed: one row of tiles per sequence
        p.vl = *a.vl;
        grid = dim3((unsigned)tiles, (unsigned)a.vl->S);
    } else {
        p.vl.S = 0;
    }
    cudaError_t e;
    if (fp8)
        e = a.qI_weight ? launch_k<true, true>(grid, tm, p, s) : launch_k<true, false>(grid, tm, p, s);
    else
        e = a.qI_weight ? launch_k<false, true>(grid, tm, p, s) : launch_k<false, false>(grid, tm, p, s);
    if (e != cudaSuccess) return e;
    count_launch();
    return cudaGetLastError();
}

}  // namespace csa
