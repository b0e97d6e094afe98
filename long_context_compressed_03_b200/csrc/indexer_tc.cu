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
// Scores: for every chunk of 32 entries the MMA warp issues one tcgen05 MMA
// per indexer head (M = 128 queries, N = 32 entries, K = 64) into TMEM;
// four epilogue warpgroups take chunks in turn (TMEM: 4 buffers x 4 heads
// x 32 columns).  Each epilogue thread owns one query row.
//
// Selection: every (row, entry) gets the unique 48-bit key
//   K = (bits of the non-negative fp32 score) << 16 | (65535 - s),
// (with gate weights the scores are signed and score_key() supplies the
// order-preserving 32 bits instead of the raw bit pattern)
// which orders like (score desc, index asc) -- the top-k tie rule.  An
// MSB-first radix select over 8-bit digits finds, per row, the digit prefix
// that holds the k-th largest key: each pass recomputes the scores (the
// tensor cores make that cheap) and histograms the next digit of the keys
// that match the row's current prefix into per-row u16 bins in shared
// memory ([bin][row] layout: conflict-free; both epilogue groups add with
// fire-and-forget shared atomics).  Once a row's boundary bin has
// at most kCap keys, a final pass writes every key above the boundary to the
// output and collects the boundary bin, which is then sorted exactly; each
// selected row is finally rewritten in ascending entry order through a
// bitmap (a deterministic order).
// The score matrix never leaves the SM.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace csa {
namespace {

using namespace tc;

constexpr int kRows = 128;      // queries per CTA = MMA M
constexpr int kN = 32;          // entries per chunk = MMA N
constexpr int kGroups = 4;      // epilogue warpgroups (one TMEM buffer each)
constexpr int kHeads = 4;       // indexer heads held in TMEM
constexpr int kDim = 64;        // indexer head dim = MMA K
constexpr int kThreads = 576;   // warp 0 TMA, warp 1 MMA, warps 2-17: four epilogue groups
constexpr int kCap = 64;        // boundary-bin capacity per row
constexpr int kLevels = 6;      // 48-bit key, 8-bit digits

template <bool FP8>
struct Cfg {
    static constexpr int kElem = FP8 ? 1 : 2;
    static constexpr int kRowBytes = kDim * kElem;                  // 64 / 128
    static constexpr int kATile = kRows * kRowBytes;                // per head
    static constexpr int kBTile = kN * kRowBytes;                   // per chunk
    static constexpr int kStages = FP8 ? 4 : 3;
    static constexpr int kKSteps = FP8 ? 2 : 4;                     // K=32 (fp8) / 16 (bf16)
    static constexpr int kHist = 256 * kRows * 4;                   // u32 bins, both groups
    static constexpr size_t kSmem = 1024 + kHeads * kATile + kStages * kBTile + kHist + 8192;
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
    const int* n_entries;
    int* idx_out;
    uint32_t* err;
    VarlenMap vl;              // packed sequences (vl.S > 0): grid.y = sequence
};

struct __align__(8) Ctrl {
    uint64_t full[4];
    uint64_t freeb[4];
    uint64_t acc_full[kGroups];
    uint64_t acc_free[kGroups];
    uint64_t fin;
    uint32_t tmem_base;
    int abort;
    int next_emit;             // 1: the next pass emits
};

// Per-row selection state (shared by both epilogue groups).
struct RowState {
    uint64_t prefix[kRows];    // key prefix above the current digit
    int level[kRows];          // digit being histogrammed (or, when ready, the last one)
    int rank[kRows];           // keys still needed from the prefix's bin
    int ready[kRows];          // boundary bin small enough (or keys unique)
    int V[kRows];              // visible entries (0 for rows beyond n)
    int emitted[kRows];        // output slots used
    int listed[kRows];         // boundary keys collected
    float qs[kRows][kHeads];   // per-head query scales
};

__device__ __forceinline__ int shift_of(int level) { return 40 - 8 * level; }

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

enum PassKind { kHist0 = 0, kHist32 = 1, kHist64 = 2, kEmit = 3 };

struct RowCtx {
    int V;
    uint64_t prefix;
    int sh;
    uint32_t* hrow;
    int* orow;
    uint64_t* list;
    int* emitted;
    int* listed;
    int topk;
    float qs[kHeads];
};

// Four heads x 8 columns (head h at column offset h*kN) with one wait.
__device__ __forceinline__ void tmem_ld8x4(uint32_t taddr, float (*v)[8]) {
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

// One score of this thread's row: fold the four heads, then histogram or
// emit its key according to the row's pass kind.  KIND_T < 0 takes the kind
// at run time (rows of one warp at different radix levels).
template <bool FP8, bool GATED, int KIND_T>
__device__ __forceinline__ void score_one(const float (&acc)[kHeads][8], int e, float ks, int s,
                                          int kind_rt, const RowCtx& rc) {
    const int KIND = KIND_T >= 0 ? KIND_T : kind_rt;
    // a + |a| = 2 ReLU(a) exactly (+0 for a <= 0), and rc.qs holds qs / 2
    // (times the gate weight), so this is sum_h qs_h ReLU(a_h) on the FMA
    // pipe: +0 or positive without weights, of any sign with them
    float sc = rc.qs[0] * (acc[0][e] + fabsf(acc[0][e]));
#pragma unroll
    for (int h = 1; h < kHeads; ++h) sc = fmaf(rc.qs[h], acc[h][e] + fabsf(acc[h][e]), sc);
    if (FP8) sc *= ks;
    const uint32_t sbits = GATED ? score_key(sc) : __float_as_uint(sc);
    if (KIND == kHist0) {
        atomicAdd(rc.hrow + (sbits >> 24) * kRows, 1u);
    } else if (KIND == kHist32) {
        const int sh32 = rc.sh - 16;
        if ((sbits >> (sh32 + 8)) == (uint32_t)rc.prefix)
            atomicAdd(rc.hrow + ((sbits >> sh32) & 255u) * kRows, 1u);
    } else {
        const uint64_t key = ((uint64_t)sbits << 16) | (uint64_t)(65535 - s);
        if (KIND == kHist64) {
            if ((key >> (rc.sh + 8)) == rc.prefix)
                atomicAdd(rc.hrow + ((key >> rc.sh) & 255u) * kRows, 1u);
        } else {
            const uint64_t kp = key >> rc.sh;
            if (kp > rc.prefix) {
                const int pos = atomicAdd(rc.emitted, 1);
                if (pos < rc.topk) rc.orow[pos] = s;
            } else if (kp == rc.prefix) {
                const int pos = atomicAdd(rc.listed, 1);
                if (pos < kCap) rc.list[pos] = key;
            }
        }
    }
}

// One chunk of 32 entries for this thread's row.  The TMEM loads and the
// scale broadcasts are .sync.aligned / warp-collective: every lane of the
// warp runs them at the same point, before any per-row branching; rows that
// are not selecting skip the arithmetic.  KIND_T >= 0 when every selecting
// row of the warp is in the same pass kind (the usual case).
template <bool FP8, bool GATED, int KIND_T>
__device__ __forceinline__ void chunk_pass(uint32_t taddr, float ksv, int c, bool active,
                                           int kind_rt, const RowCtx& rc) {
#pragma unroll 1
    for (int part = 0; part < kN / 8; ++part) {
        float acc[kHeads][8];
        tmem_ld8x4(taddr + part * 8, acc);
        // lane e of the warp holds the key scale of entry c*kN + e: broadcast
        // the part's eight before any per-row branching (warp-collective)
        float ks[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ks[e] = FP8 ? __shfl_sync(0xffffffffu, ksv, part * 8 + e) : 1.0f;
        if (!active) continue;
        const int s0 = c * kN + part * 8;
        if (s0 + 8 <= rc.V) {
#pragma unroll
            for (int e = 0; e < 8; ++e) score_one<FP8, GATED, KIND_T>(acc, e, ks[e], s0 + e, kind_rt, rc);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (s0 + e < rc.V) score_one<FP8, GATED, KIND_T>(acc, e, ks[e], s0 + e, kind_rt, rc);
        }
    }
}

template <bool FP8, bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tm_k, IdxParams p) {
    using C = Cfg<FP8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;                                       // [kHeads][kATile]
    uint8_t* sB = sA + kHeads * C::kATile;                    // [kStages][kBTile]
    uint32_t* hist = reinterpret_cast<uint32_t*>(sB + C::kStages * C::kBTile);   // [256][128]
    uint64_t* list = reinterpret_cast<uint64_t*>(hist);      // [128][kCap] (aliases hist)
    RowState* rs = reinterpret_cast<RowState*>(reinterpret_cast<uint8_t*>(hist) + C::kHist);
    Ctrl* ctl = reinterpret_cast<Ctrl*>(reinterpret_cast<uint8_t*>(rs) + sizeof(RowState));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's 128 queries: element (or packed sequence) b, positions
    // t0 .. of its slen; its rows start at token tok0 and entry ent0.  Heavy
    // tiles (late queries see more entries) first.
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
    const int Vmax = min((t_last + 1) / p.m, ne);
    const int nchunks = (Vmax + kN - 1) / kN;
    volatile int* abort = &ctl->abort;

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->freeb[s], 1);
        }
        for (int g = 0; g < kGroups; ++g) {
            mbar_init(&ctl->acc_full[g], 1);
            mbar_init(&ctl->acc_free[g], kRows);
        }
        mbar_init(&ctl->fin, 1);
        ctl->abort = (*reinterpret_cast<volatile uint32_t*>(p.err) != 0u) ? 1 : 0;
        ctl->next_emit = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, 512);
        tmem_relinquish();
    }
    // rows: visibility and the query operand (one warp per (row, head) pair)
    for (int r = threadIdx.x; r < kRows; r += kThreads) {
        const int t = t0 + r;
        const int V = (t < slen) ? min((t + 1) / p.m, ne) : 0;
        rs->V[r] = V;
        rs->level[r] = 0;
        rs->prefix[r] = 0;
        rs->rank[r] = p.topk;
        rs->ready[r] = (V <= p.topk) ? 1 : 0;   // rows with V <= k take every visible entry
        rs->emitted[r] = 0;
        rs->listed[r] = 0;
    }
    for (int pair = warp; pair < kRows * kHeads; pair += kThreads / 32) {
        const int r = pair >> 2, h = pair & 3;
        const int t = min(t0 + r, slen - 1);
        const size_t qrow = (tok0 + t) * p.H_I + h;
        float v0 = 0.0f, v1 = 0.0f;   // elements 2*lane, 2*lane+1
        float qs = 1.0f;
        uint32_t packed;              // two output elements (fp8: 2 bytes; bf16: 4 bytes)
        if (h < p.H_I) {
            if (p.q_mode == 2) {
                const uint8_t* src = static_cast<const uint8_t*>(p.qI) + qrow * kDim;
                packed = (uint32_t)src[2 * lane] | ((uint32_t)src[2 * lane + 1] << 8);
                qs = p.qI_scale[qrow];
            } else {
                const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(p.qI) + qrow * kDim;
                v0 = __bfloat162float(src[2 * lane]);
                v1 = __bfloat162float(src[2 * lane + 1]);
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
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(v0, v1);
                    packed = *reinterpret_cast<uint32_t*>(&h2);
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
        if (GATED && h < p.H_I) qs *= p.qw[qrow];
        if (lane == 0) rs->qs[r][h] = (h < p.H_I) ? qs : 0.0f;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    // any row that needs selection at all?
    int need = 0;
    for (int r = 0; r < kRows; ++r) need |= (rs->ready[r] == 0);

    // role counters that persist across passes
    int L = 0;                 // producer / MMA: chunk loads issued
    int use_buf[kGroups] = {0, 0, 0, 0};   // MMA: issues into each TMEM buffer
    int cons = 0;              // epilogue: chunks consumed by this group
    const bool is_epi = warp >= 2;
    const int grp = is_epi ? ((warp - 2) >> 2) : 0;      // warps 2-5, 6-9, 10-13, 14-17
    const int r = (warp & 3) * 32 + lane;                    // epilogue row
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;

    for (int pass = 0; need && pass <= kLevels; ++pass) {
        const bool emit = ctl->next_emit != 0;
        if (!emit) {
            for (int i = threadIdx.x; i < 256 * kRows; i += kThreads) hist[i] = 0u;
        }
        __syncthreads();
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                for (int c = 0; c < nchunks; ++c, ++L) {
                    const int slot = L % C::kStages, u = L / C::kStages;
                    if (*abort) break;     // nothing is issued once the CTA aborts
                    if (u > 0 && !mbar_wait(&ctl->freeb[slot], (u - 1) & 1, abort, p.err)) break;
                    mbar_arrive_expect_tx(&ctl->full[slot], C::kBTile);
                    tma_load_2d(sB + slot * C::kBTile, &tm_k, 0, (int)ent0 + c * kN, &ctl->full[slot]);
                }
            }
            __syncwarp();
            L = __shfl_sync(0xffffffffu, L, 0);
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                const uint32_t idesc = FP8 ? idesc_e4m3(kRows, kN) : idesc_bf16(kRows, kN, false, false);
                for (int c = 0; c < nchunks; ++c, ++L) {
                    const int slot = L % C::kStages;
                    const int g = c % kGroups;
                    if (!mbar_wait(&ctl->full[slot], (L / C::kStages) & 1, abort, p.err)) break;
                    if (use_buf[g] > 0 && !mbar_wait(&ctl->acc_free[g], (use_buf[g] - 1) & 1, abort, p.err)) break;
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
                                mma_f8_ss(tmem + g * 128 + h * kN, ad, bd, idesc, k > 0);
                            else
                                mma_bf16_ss(tmem + g * 128 + h * kN, ad, bd, idesc, k > 0);
                        }
                    }
                    mma_commit(&ctl->acc_full[g]);
                    mma_commit(&ctl->freeb[slot]);
                    ++use_buf[g];
                }
            }
            __syncwarp();
            L = __shfl_sync(0xffffffffu, L, 0);
            for (int g = 0; g < kGroups; ++g) use_buf[g] = __shfl_sync(0xffffffffu, use_buf[g], 0);
        } else {
            // ------------------------------------------------------------ epilogue
            const int V = rs->V[r];
            const bool row_ok = t0 + r < slen;
            const bool active = row_ok && V > p.topk && (rs->ready[r] == 0 || emit);
            const int level = rs->level[r];
            const int kind = emit ? kEmit : (level == 0 ? kHist0 : (level < 4 ? kHist32 : kHist64));
            RowCtx rc;
            rc.V = V;
            rc.prefix = rs->prefix[r];
            rc.sh = shift_of(level);
            rc.hrow = hist + r;
            rc.orow = p.idx_out + (tok0 + min(t0 + r, slen - 1)) * p.topk;
            rc.list = list + r * kCap;
            rc.emitted = &rs->emitted[r];
            rc.listed = &rs->listed[r];
            rc.topk = p.topk;
#pragma unroll
            for (int h = 0; h < kHeads; ++h) rc.qs[h] = 0.5f * rs->qs[r][h];   // exact: a power of two
            const float* ksc = FP8 ? p.kI_scale + ent0 : nullptr;
            // this lane's key scale for entry c*kN + lane, loaded one chunk ahead
            auto scale_of = [&](int c) -> float {
                const int e = c * kN + lane;
                return (FP8 && c < nchunks && e < Vmax) ? __ldg(ksc + e) : 0.0f;
            };
            float ksv = scale_of(grp);
            // the pass kind shared by every selecting row of the warp, or -1
            const uint32_t act = __ballot_sync(0xffffffffu, active);
            const int k0 = __shfl_sync(0xffffffffu, kind, act ? __ffs(act) - 1 : 0);
            const int wkind = __all_sync(0xffffffffu, !active || kind == k0) ? k0 : -1;
            for (int c = grp; c < nchunks; c += kGroups) {
                const float ksv_next = scale_of(c + kGroups);
                if (!__all_sync(0xffffffffu, mbar_wait(&ctl->acc_full[grp], cons & 1, abort, p.err))) break;
                tc_fence_after();
                const uint32_t taddr = tmem + lane_addr + grp * 128;
                switch (wkind) {
                    case kHist0: chunk_pass<FP8, GATED, kHist0>(taddr, ksv, c, active, kind, rc); break;
                    case kHist32: chunk_pass<FP8, GATED, kHist32>(taddr, ksv, c, active, kind, rc); break;
                    case kHist64: chunk_pass<FP8, GATED, kHist64>(taddr, ksv, c, active, kind, rc); break;
                    case kEmit: chunk_pass<FP8, GATED, kEmit>(taddr, ksv, c, active, kind, rc); break;
                    default: chunk_pass<FP8, GATED, -1>(taddr, ksv, c, active, kind, rc); break;
                }
                ksv = ksv_next;
                tc_fence_before();
                mbar_arrive(&ctl->acc_free[grp]);
                ++cons;
            }
        }
        __syncthreads();
        if (*abort) break;
        // ---------------------------------------------------------------- per-row bookkeeping
        if (is_epi && grp == 0) {
            const int V = rs->V[r];
            if (!emit) {
                if (!rs->ready[r] && V > p.topk) {
                    // merge the two groups' bins; find the digit holding rank
                    int rank = rs->rank[r];
                    int run = 0, digit = 0, inbin = 0;
                    for (int d = 255; d >= 0; --d) {
                        const int cnt = (int)hist[d * kRows + r];
                        if (run + cnt >= rank) { digit = d; inbin = cnt; break; }
                        run += cnt;
                    }
                    const int level = rs->level[r];
                    rs->prefix[r] = (rs->prefix[r] << 8) | (uint64_t)digit;
                    rs->rank[r] = rank - run;
                    if (inbin <= kCap || level == kLevels - 1) {
                        rs->ready[r] = 1;          // emit with this prefix at this level's shift
                    } else {
                        rs->level[r] = level + 1;
                    }
                }
            } else if (t0 + r < slen) {
                int* orow = p.idx_out + (tok0 + t0 + r) * p.topk;
                if (V <= p.topk) {
                    for (int j = 0; j < p.topk; ++j) orow[j] = j < V ? j : -1;
                } else {
                    // boundary keys: the rank largest, by insertion into a sorted prefix
                    const int nl = min(rs->listed[r], kCap);
                    uint64_t* lr = list + r * kCap;
                    for (int i = 1; i < nl; ++i) {
                        const uint64_t v = lr[i];
                        int j = i - 1;
                        while (j >= 0 && lr[j] < v) { lr[j + 1] = lr[j]; --j; }
                        lr[j + 1] = v;
                    }
                    int pos = min(rs->emitted[r], p.topk);
                    const int want = min(rs->rank[r], nl);
                    for (int i = 0; i < want && pos < p.topk; ++i, ++pos)
                        orow[pos] = 65535 - (int)(lr[i] & 0xFFFFu);
                    for (; pos < p.topk; ++pos) orow[pos] = -1;   // unreachable when counts agree
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
                const int ew = warp - 2;
                uint32_t* bm = hist + ew * 2048;                 // 8 KB per warp: V <= 65536
                const int kk = p.topk;
                for (int rr = ew; rr < kRows; rr += kGroups * 4) {
                    const int V = rs->V[rr];
                    if (t0 + rr >= slen || V <= kk) continue;
                    int* orow = p.idx_out + (tok0 + t0 + rr) * kk;
                    const int nw = (V + 31) >> 5;
                    for (int i = lane; i < nw; i += 32) bm[i] = 0u;
                    __syncwarp();
                    for (int i = lane; i < kk; i += 32) {
                        const int sidx = orow[i];
                        if (sidx >= 0 && sidx < V) atomicOr(&bm[sidx >> 5], 1u << (sidx & 31));
                    }
                    __syncwarp();
                    int basepos = 0;
                    for (int w0 = 0; w0 < nw; w0 += 32) {
                        uint32_t word = (w0 + lane < nw) ? bm[w0 + lane] : 0u;
                        const int cnt = __popc(word);
                        int incl = cnt;
#pragma unroll
                        for (int off = 1; off < 32; off <<= 1) {
                            const int v = __shfl_up_sync(0xffffffffu, incl, off);
                            if (lane >= off) incl += v;
                        }
                        int pos = basepos + incl - cnt;
                        while (word) {
                            const int bit = __ffs(word) - 1;
                            word &= word - 1u;
                            if (pos < kk) orow[pos] = ((w0 + lane) << 5) + bit;
                            ++pos;
                        }
                        basepos += __shfl_sync(0xffffffffu, incl, 31);
                    }
                    __syncwarp();
                }
            }
            break;
        }
        // the next pass emits once every selecting row is ready
        if (threadIdx.x == 0) {
            int all_ready = 1;
            for (int i = 0; i < kRows; ++i) all_ready &= rs->ready[i];
            ctl->next_emit = all_ready;
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
        // every row takes all its visible entries
        for (int i = threadIdx.x; i < kRows; i += kThreads) {
            if (t0 + i >= slen) continue;
            int* orow = p.idx_out + (tok0 + t0 + i) * p.topk;
            const int V = rs->V[i];
            for (int j = 0; j < p.topk; ++j) orow[j] = j < V ? j : -1;
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
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg<FP8>::kSmem);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, Cfg<FP8>::kSmem, s>>>(tm, p);
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
    p.err = err;
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
