// attention_tc.cu -- tensor-core (tcgen05) prefill attention for the CSA /
// HCA joint softmax with 64 query heads of dimension 128 sharing one KV head.
//
// For query token t and head h (one softmax over the multiset union):
//   keys = compressed set(t) ∪ raw window [max(0, t-W+1), t]
//   o = sum softmax(scale * q.key) key          (key = value: shared-KV MQA)
// ("DS-V4 分析&学习" §1.2, §1.4, §1.5; "百万上下文从「奢侈品」变「日用品」…"
//  §4.3, §5.2.)  Compressed set: the token's top-k entries (sparse mode) or
// every entry s < floor((t+1)/m) (dense / HCA mode).
//
// Work unit: one CTA owns 4 consecutive tokens of one sequence as two M=128
// tiles (2 tokens x 64 heads each).  Every head of a token attends to the
// same keys, so a key tile of 128 rows x 128 dims serves a whole M tile.
//   - window tiles (and dense-mode prefix tiles) are shared by both M tiles
//     and loaded once per CTA by 2D TMA;
//   - sparse-mode compressed tiles belong to one token: their rows are
//     gathered with 16-byte cp.async copies by 128 loader threads straight
//     into the 128-byte-swizzled layout the tensor core reads (many
//     independent requests in flight), and the rows of the other token in
//     the M tile are masked.
// Roles (21 warps): warps 0-3 load (contiguous tiles by TMA; the sparse
// rows by cp.async, 16 lanes per 256-byte row, from index rows staged in
// shared memory), warp 4 allocates TMEM, loads Q by TMA and one lane issues
// every MMA, warps 5-8 / 9-12 run the softmax of M tile 0 / 1 (a warp
// reaches TMEM lanes 32*(warp%4) .. +31, so each group covers all 128
// rows), warps 13-16 / 17-20 write the output of M tile 0 / 1.
// TMEM: S0 [cols 0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// S = Q K^T (M=128, N<=128, K=128 in 8 steps), P = exp2(S*scale*log2e - m)
// written back over S as two bf16 halves (hi = bf16(P), lo = bf16(P - hi)),
// O += P_hi V + P_lo V with P read from tensor memory and V the same shared
// tile read as an MN-major operand.  The running sum adds the weights the
// MMA actually multiplies (hi + lo, about 16 significant bits), so the
// result is an exact convex combination of the keys under those weights.  The running max
// is only raised (and O rescaled in TMEM) when it grows by more than 2^8, so
// most tiles need no rescale; the final division by the running sum is exact.
#include <cudaTypedefs.h>

#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace csa {
namespace {

using namespace tc;

constexpr int kH = 64;
constexpr int kD = 128;
constexpr int kRows = 128;          // rows of an M tile
constexpr int kTokens = 4;          // tokens per CTA
constexpr int kBN = 128;            // keys per tile
constexpr int kStages = 4;
#ifndef CSA_ATTN_LOAD_WARPS
#define CSA_ATTN_LOAD_WARPS 4
#endif
constexpr int kLoadWarps = CSA_ATTN_LOAD_WARPS;   // loaders (TMA + cp.async row gathers)
constexpr int kLoadThreads = kLoadWarps * 32;
constexpr int kMmaWarp = kLoadWarps;               // TMEM allocation, MMA issue, Q loads
constexpr int kSoftWarp0 = kLoadWarps + 1;         // 4 + 4 softmax warps for M tiles 0 / 1
constexpr int kEpiWarp0 = kSoftWarp0 + 8;          // 4 + 4 epilogue warps for M tiles 0 / 1
constexpr int kThreads = (kLoadWarps + 17) * 32;
static_assert(kLoadThreads >= 128 && kLoadThreads % 128 == 0, "loaders cover the 128 rows of a tile");
constexpr int kHalf = 16384;        // one 64-column half of a 128-row tile
constexpr int kTileBytes = 32768;   // 128 rows x 128 bf16
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;


struct __align__(8) Ctrl {
    uint64_t bar_q;
    uint64_t q_free;                // the unit's last QK has read Q
    uint64_t o_full[2];             // the unit's last P.V has landed in O
    uint64_t o_free[2];             // the epilogue has read O
    uint64_t stats_ready[2];        // the softmax has published the unit's row statistics
    uint64_t full[kStages];
    uint64_t freeb[kStages];
    uint64_t s_full[2];
    uint64_t p_ready[2];
    uint64_t fin;
    uint32_t mask[kStages][4];      // gathered tiles: valid rows of the stage
    uint32_t tmem_base;
    int abort;
    int load_go;               // loaders: continue with the next load
};

struct RowStat {            // per row of an M tile at the end of a unit
    float m, lr, le;
};
constexpr size_t kStatBytes = sizeof(RowStat) * 2 /*unit parity*/ * 2 /*M tiles*/ * kRows;
constexpr size_t kSmemFixed = 1024 /*align slack*/ + 2 * kTileBytes /*Q*/ +
                              kStages * kTileBytes + sizeof(Ctrl) + kStatBytes;
// + the CTA's index rows (sparse mode): kTokens * topk int32

struct TcParams {
    const void* kv_c;          // sparse: [B, N_cap, 128] bf16 (rows gathered by cp.async)
    const int* idx;            // sparse: [B, n, topk]
    int topk;
    const int* n_entries;      // dense
    int m;
    int dense;
    int B, n, N_cap, L_raw, window;
    float scale_log2;          // softmax scale * log2(e)
    __nv_bfloat16* out;
    float* lse;
    uint32_t* err;
    VarlenMap vl;              // packed sequences (vl.S > 0)
};

struct Geometry {
    int cc;        // sparse: chunks of 128 in a token's index row
    int Tc;        // compressed tiles per M tile
    int Tw;        // window tiles
    int T;         // tiles per M tile
    int bn_c_last; // N of the last compressed tile
    int bn_w_last;
    int p_lo;      // first window position
    int Lw;
    int Vmax;      // dense: entries needed by the CTA's last token
};

__device__ __forceinline__ int round16(int v) { return (v + 15) & ~15; }

// 2^x with the MUFU instruction (ex2.approx of -inf is +0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Units of work: unit u covers tokens [t0, t0 + 4) of sequence b, where
// u = b * units_per_seq + t0 / 4 (packed sequences: u = uoff[b] + t0 / 4).
// The kernel is persistent: CTA c takes units c, c + gridDim.x, ... in that
// order, and every role walks the same list, so barrier phases run on across
// units.  A unit also carries where its sequence's rows start.
struct Unit {
    int b, t0;
    int n;          // the sequence's length
    int N;          // its compressed entries
    int L_raw;      // its raw rows
    int ne_dense;   // dense: entries it may see (n_entries, clamped)
    int tok0;       // row of its token 0 in q / out / lse / idx
    int ent0;       // row of its entry 0 in kv_c
    int raw0;       // row of its raw position 0 in kv_raw
};
template <bool PACKED>
__device__ __forceinline__ Unit unit_of(const TcParams& p, int u) {
    Unit r;
    if constexpr (PACKED) {
        int lo = 0, hi = p.vl.S - 1;                  // the last sequence with uoff <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.vl.uoff[mid] <= u) lo = mid; else hi = mid - 1;
        }
        r.b = lo;
        r.t0 = (u - p.vl.uoff[lo]) * kTokens;
        r.n = p.vl.tok[lo + 1] - p.vl.tok[lo];
        r.N = r.n / p.m;
        r.L_raw = r.n;
        r.ne_dense = r.N;
        r.tok0 = p.vl.tok[lo];
        r.ent0 = p.vl.ent[lo];
        r.raw0 = r.tok0;
    } else {
        // the other fields are derived from p and b where they are used
        // (accessors below), so nothing extra stays live in registers
        const int per = (p.n + kTokens - 1) / kTokens;
        r.b = u / per;
        r.t0 = (u - r.b * per) * kTokens;
    }
    return r;
}

// A unit's fields: stored for packed sequences, derived from the call's
// uniform shape otherwise.
template <bool PACKED> __device__ __forceinline__ int u_n(const TcParams& p, const Unit& u) {
    return PACKED ? u.n : p.n;
}
template <bool PACKED> __device__ __forceinline__ int u_N(const TcParams& p, const Unit& u) {
    return PACKED ? u.N : p.N_cap;
}
template <bool PACKED> __device__ __forceinline__ int u_L_raw(const TcParams& p, const Unit& u) {
    return PACKED ? u.L_raw : p.L_raw;
}
template <bool PACKED> __device__ __forceinline__ int u_ne_dense(const TcParams& p, const Unit& u) {
    return PACKED ? u.ne_dense : clampi(p.n_entries ? p.n_entries[u.b] : p.N_cap, 0, p.N_cap);
}
template <bool PACKED> __device__ __forceinline__ int u_tok0(const TcParams& p, const Unit& u) {
    return PACKED ? u.tok0 : u.b * p.n;
}
template <bool PACKED> __device__ __forceinline__ int u_ent0(const TcParams& p, const Unit& u) {
    return PACKED ? u.ent0 : u.b * p.N_cap;
}
template <bool PACKED> __device__ __forceinline__ int u_raw0(const TcParams& p, const Unit& u) {
    return PACKED ? u.raw0 : u.b * p.L_raw;
}

template <bool PACKED>
__device__ __forceinline__ Geometry geometry(const TcParams& p, const Unit& un) {
    Geometry g;
    const int t0 = un.t0;
    const int t_last = min(t0 + kTokens - 1, u_n<PACKED>(p, un) - 1);
    if (p.dense) {
        g.Vmax = min((t_last + 1) / p.m, u_ne_dense<PACKED>(p, un));
        g.cc = 0;
        g.Tc = (g.Vmax + kBN - 1) / kBN;
        g.bn_c_last = g.Tc ? round16(g.Vmax - (g.Tc - 1) * kBN) : 0;
    } else {
        g.Vmax = 0;
        const int cc = (p.topk + kBN - 1) / kBN;
        g.cc = cc;
        g.Tc = 2 * cc;
        g.bn_c_last = p.topk ? round16(p.topk - (cc - 1) * kBN) : 0;
    }
    if (p.window > 0) {
        g.p_lo = max(0, t0 - p.window + 1);
        const int p_hi = min(t_last, u_L_raw<PACKED>(p, un) - 1);
        g.Lw = max(0, p_hi - g.p_lo + 1);
    } else {
        g.p_lo = 0;
        g.Lw = 0;
    }
    g.Tw = (g.Lw + kBN - 1) / kBN;
    g.bn_w_last = g.Tw ? round16(g.Lw - (g.Tw - 1) * kBN) : 0;
    g.T = g.Tc + g.Tw;
    return g;
}

// Tile j of M tile mt: which load carries it, and its N size.
struct TileRef {
    int load;
    int bn;
    int kind;   // 0 gathered (sparse compressed), 1 dense prefix, 2 window
    int token;  // gathered: token (0/1) of the M tile the rows belong to
    int chunk;  // gathered: chunk of the token's index row; contiguous: tile index in segment
    bool last_consumer;
};

__device__ __forceinline__ TileRef tile_ref(const TcParams& p, const Geometry& g, int mt, int j) {
    TileRef r;
    if (j < g.Tc) {
        if (p.dense) {
            r.load = j;
            r.kind = 1;
            r.chunk = j;
            r.token = 0;
            r.bn = (j == g.Tc - 1) ? g.bn_c_last : kBN;
            r.last_consumer = (mt == 1);
        } else {
            const int cc = g.cc;
            r.load = 2 * j + mt;
            r.kind = 0;
            r.token = j / cc;
            r.chunk = j % cc;
            r.bn = (r.chunk == cc - 1) ? g.bn_c_last : kBN;
            r.last_consumer = true;
        }
    } else {
        const int jw = j - g.Tc;
        r.load = (p.dense ? g.Tc : 2 * g.Tc) + jw;
        r.kind = 2;
        r.token = 0;
        r.chunk = jw;
        r.bn = (jw == g.Tw - 1) ? g.bn_w_last : kBN;
        r.last_consumer = (mt == 1);
    }
    return r;
}

__device__ __forceinline__ int total_loads(const TcParams& p, const Geometry& g) {
    return (p.dense ? g.Tc : 2 * g.Tc) + g.Tw;
}

// Valid-column bits of a 128-key tile for one row: columns [c_lo, c_hi]
// intersected with the gathered-row mask gm.
__device__ __forceinline__ void valid_bits(int c_lo, int c_hi, const uint32_t gm[4], uint32_t vm[4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int lo = max(c_lo - 32 * q, 0), hi = min(c_hi - 32 * q, 31);
        vm[q] = (lo > hi) ? 0u : ((0xffffffffu >> (31 - hi)) & (0xffffffffu << lo)) & gm[q];
    }
}

// Row max (base-2 scaled) of the valid columns of this thread's S row.
__device__ __forceinline__ float tile_max(uint32_t s_addr, const uint32_t vm[4], float sl2) {
    float mx = -INFINITY;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        const uint32_t mq = q == 0 ? vm[0] : (q == 1 ? vm[1] : (q == 2 ? vm[2] : vm[3]));
        float sv[32];
        tmem_ld32(s_addr + q * 32, sv);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float z = ((mq >> i) & 1u) ? sv[i] * sl2 : -INFINITY;
            mx = fmaxf(mx, z);
        }
    }
    return mx;
}

// The weight p of a key goes to the P.V product as two bf16 numbers,
// hi = bf16(p) and lo = bf16(p - hi), whose sum carries about 16 significant
// bits: a single bf16 weight (8 bits) moves the output by up to 2^-8 of the
// spread of the values it averages, which for keys of magnitude ~16 is
// several 1e-2.  hi + lo is exact in fp32.
__device__ __forceinline__ void split_bf16(float p0, float p1, uint32_t& hi, uint32_t& lo, float& h0,
                                           float& h1, float& s0, float& s1) {
    __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
    hi = *reinterpret_cast<uint32_t*>(&hb);
    h0 = __uint_as_float(hi << 16);
    h1 = __uint_as_float(hi & 0xffff0000u);
    __nv_bfloat162 lb = __floats2bfloat162_rn(p0 - h0, p1 - h1);
    lo = *reinterpret_cast<uint32_t*>(&lb);
    s0 = h0 + __uint_as_float(lo << 16);
    s1 = h1 + __uint_as_float(lo & 0xffff0000u);
}

// P row = exp2(z - m) for the valid columns (0 elsewhere), written over S as
// it goes: chunk q reads S columns [32q, 32q+32) and writes the chunk's hi
// weights (bf16 pairs) to columns [32q, 32q+16) and its lo weights to
// [32q+16, 32q+32), which it has just read.  Accumulates the exact sum and
// the sum of the weights the MMA multiplies (hi + lo).  m = +inf writes an
// all-zero row.
__device__ __forceinline__ void tile_exp(uint32_t s_addr, const uint32_t vm[4], float sl2, float m,
                                         float& se, float& sr) {
    // kept rolled: unrolling lets the compiler interleave chunks past the
    // register budget
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        const uint32_t mq = q == 0 ? vm[0] : (q == 1 ? vm[1] : (q == 2 ? vm[2] : vm[3]));
        float sv[32];
        tmem_ld32(s_addr + q * 32, sv);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t pk[8], pl[8];
#pragma unroll
            for (int e = 16 * hh; e < 16 * hh + 16; e += 2) {
                const float z0 = ((mq >> e) & 1u) ? sv[e] * sl2 : -INFINITY;
                const float z1 = ((mq >> (e + 1)) & 1u) ? sv[e + 1] * sl2 : -INFINITY;
                const float p0 = ex2(z0 - m), p1 = ex2(z1 - m);
                float h0, h1, s0, s1;
                split_bf16(p0, p1, pk[(e >> 1) & 7], pl[(e >> 1) & 7], h0, h1, s0, s1);
                se += p0 + p1;
                sr += s0 + s1;
            }
            tmem_st8(s_addr + q * 32 + 8 * hh, pk);
            tmem_st8(s_addr + q * 32 + 16 + 8 * hh, pl);
        }
    }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// tile_max for a row whose 128 columns are all keys: the max of S, scaled
// once (the scale is positive, so the maximum element is the same).
__device__ __forceinline__ float tile_max_full(uint32_t s_addr, float sl2) {
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        float sv[32];
        tmem_ld32(s_addr + q * 32, sv);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            mx0 = max3(mx0, sv[i], sv[i + 1]);
            mx1 = max3(mx1, sv[i + 2], sv[i + 3]);
        }
    }
    return fmaxf(mx0, mx1) * sl2;
}

// tile_exp for a row whose 128 columns are all keys, on packed f32x2 math:
// z = S * scale - m in one rounding, P = 2^z, the rounded weights summed in
// pairs; the exact sum only when the log-sum-exp is wanted.
__device__ __forceinline__ void tile_exp_full(uint32_t s_addr, float sl2, float m, bool want_se,
                                              float& se, float& sr) {
    const uint64_t sl2x2 = f2_pack(sl2, sl2), negm = f2_pack(-m, -m);
    uint64_t accr = 0, acce = 0;      // (+0, +0)
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        float sv[32];
        tmem_ld32(s_addr + q * 32, sv);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t pk[8], pl[8];
#pragma unroll
            for (int e = 16 * hh; e < 16 * hh + 16; e += 2) {
                const uint64_t z = f2_fma(f2_pack(sv[e], sv[e + 1]), sl2x2, negm);
                const float p0 = ex2(__uint_as_float((uint32_t)z)), p1 = ex2(__uint_as_float((uint32_t)(z >> 32)));
                float h0, h1, s0, s1;
                split_bf16(p0, p1, pk[(e >> 1) & 7], pl[(e >> 1) & 7], h0, h1, s0, s1);
                accr = f2_add(accr, f2_pack(s0, s1));
                if (want_se) acce = f2_add(acce, f2_pack(p0, p1));
            }
            tmem_st8(s_addr + q * 32 + 8 * hh, pk);
            tmem_st8(s_addr + q * 32 + 16 + 8 * hh, pl);
        }
    }
    sr += __uint_as_float((uint32_t)accr) + __uint_as_float((uint32_t)(accr >> 32));
    se += __uint_as_float((uint32_t)acce) + __uint_as_float((uint32_t)(acce >> 32));
}

// The row max rose by more than 2^8 (or a row sees its first keys): rescale
// the sums and O.  alpha = 0 for a row without earlier keys.
__device__ __noinline__ void rescale_o(uint32_t o_addr, float alpha) {
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        float ov[32];
        tmem_ld32(o_addr + q * 32, ov);
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] *= alpha;
        tmem_st32(o_addr + q * 32, ov);
    }
    tmem_st_wait();
}

// 21 warps sit on the SM's four 16,384-register partitions as 6 + 5 + 5 + 5,
// so a thread may hold at most 80 registers (6 x 32 x 80 = 15,360).
template <bool PACKED>
__global__ void __maxnreg__(80)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_c,
               const __grid_constant__ CUtensorMap tm_w, TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = base;                                  // [2][32 KB]
    uint8_t* sK = sQ + 2 * kTileBytes;                   // [kStages][32 KB]
    Ctrl* ctl = reinterpret_cast<Ctrl*>(sK + kStages * kTileBytes);
    RowStat* stats = reinterpret_cast<RowStat*>(ctl + 1);        // [2][2][kRows]
    int* sIdx = reinterpret_cast<int*>(stats + 4 * kRows);       // [kTokens][topk]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_units = PACKED ? p.vl.uoff[p.vl.S] : p.B * ((p.n + kTokens - 1) / kTokens);
    volatile int* abort = &ctl->abort;

    if (threadIdx.x == 0) {
        mbar_init(&ctl->bar_q, 1);
        mbar_init(&ctl->q_free, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl->full[s], kLoadThreads + 1);
            mbar_init(&ctl->freeb[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->s_full[i], 1);
            mbar_init(&ctl->p_ready[i], kRows);
            mbar_init(&ctl->o_full[i], 1);
            mbar_init(&ctl->o_free[i], kRows);
            mbar_init(&ctl->stats_ready[i], kRows);
        }
        mbar_init(&ctl->fin, 1);
        // a CTA started after another one timed out does no work
        ctl->abort = (*reinterpret_cast<volatile uint32_t*>(p.err) != 0u) ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&ctl->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    if (warp < kLoadThreads / 32) {
        // ------------------------------------------------------------ loaders
        const int lt = threadIdx.x;                          // 0 .. kLoadThreads-1
        if (lt == 0) {
            prefetch_tmap(&tm_c);
            prefetch_tmap(&tm_w);
        }
        int Lg = 0;                                          // loads issued by this CTA
        bool go = true;
        for (int u = blockIdx.x; u < n_units && go; u += gridDim.x) {
            const Unit un = unit_of<PACKED>(p, u);
            const int t0 = un.t0;
            const Geometry g = geometry<PACKED>(p, un);
            // the unit's index rows (out-of-range tokens read as padding); the
            // previous unit's gathers have all been issued
            named_sync(1, kLoadThreads);
            if (!p.dense) {
                for (int i = lt; i < kTokens * p.topk; i += kLoadThreads) {
                    const int tok = i / p.topk, c = i - tok * p.topk;
                    const int t = t0 + tok;
                    sIdx[i] = (t < u_n<PACKED>(p, un)) ? __ldg(p.idx + (size_t)(u_tok0<PACKED>(p, un) + t) * p.topk + c) : -1;
                }
            }
            named_sync(1, kLoadThreads);
            const int NL = total_loads(p, g);
            const int nc = p.dense ? g.Tc : 2 * g.Tc;
            const uint8_t* kvc_rows = static_cast<const uint8_t*>(p.kv_c) + (size_t)u_ent0<PACKED>(p, un) * (kD * 2);
            for (int L = 0; L < NL; ++L, ++Lg) {
                const int slot = Lg % kStages, use = Lg / kStages;
                uint8_t* dst = sK + slot * kTileBytes;
                // which tile is load L of the unit?
                int kind, token = 0, chunk;
                if (L < nc) {
                    if (p.dense) { kind = 1; chunk = L; }
                    else {
                        const int j = L >> 1, mt = L & 1;
                        kind = 0;
                        token = 2 * mt + j / g.cc;    // token within the unit
                        chunk = j - (j / g.cc) * g.cc;
                    }
                } else {
                    kind = 2;
                    chunk = L - nc;
                }
                // one thread acquires the free slot and decides for all loaders;
                // the named barrier orders the others after it
                if (lt == 0) {
                    const bool okw = use == 0 || mbar_wait(&ctl->freeb[slot], (use - 1) & 1, abort, p.err);
                    ctl->load_go = (okw && !*abort) ? 1 : 0;
                }
                named_sync(1, kLoadThreads);
                if (!ctl->load_go) { go = false; break; }
                if (kind == 0) {
                    const int* ir = sIdx + token * p.topk + chunk * kBN;
                    const int tpos = t0 + token;
                    // valid-row mask: loader thread lt < 128 checks row lt
                    if (lt < kBN) {
                        const int c = chunk * kBN + lt;
                        const int sv = (c < p.topk) ? ir[lt] : -1;
                        const bool ok = tpos < u_n<PACKED>(p, un) && sv >= 0 && sv < u_N<PACKED>(p, un);
                        const uint32_t bits = __ballot_sync(0xffffffffu, ok);
                        if (lane == 0) ctl->mask[slot][warp] = bits;
                    }
                    // rows: 16 lanes per 256-byte row, kLoadThreads/16 rows per round
                    constexpr int kRowsPerRound = kLoadThreads / 16;
                    const int c16 = lt & 15, half = c16 >> 3, cc = c16 & 7;
#pragma unroll 4
                    for (int it = 0; it < kBN / kRowsPerRound; ++it) {
                        const int row = it * kRowsPerRound + (lt >> 4);
                        const int c = chunk * kBN + row;
                        int sv = (c < p.topk) ? ir[row] : -1;
                        if (tpos >= u_n<PACKED>(p, un) || sv < 0 || sv >= u_N<PACKED>(p, un)) sv = 0;   // masked; any valid row
                        const uint8_t* src = kvc_rows + (size_t)sv * (kD * 2) + c16 * 16;
                        cp_async16(dst + half * kHalf + row * 128 + ((cc ^ (row & 7)) << 4), src);
                    }
                    cp_async_arrive_noinc(&ctl->full[slot]);
                    named_sync(1, kLoadThreads);                 // every mask word is written
                    if (lt == 0) mbar_arrive(&ctl->full[slot]);  // releases the mask
                } else {
                    if (lt == 0) {
                        const CUtensorMap* tm = (kind == 1) ? &tm_c : &tm_w;
                        const int row = (kind == 1) ? u_ent0<PACKED>(p, un) + chunk * kBN
                                                    : u_raw0<PACKED>(p, un) + g.p_lo + chunk * kBN;
                        mbar_arrive_expect_tx(&ctl->full[slot], kTileBytes);
                        for (int h = 0; h < 2; ++h)
                            tma_load_2d(dst + h * kHalf, tm, h * 64, row, &ctl->full[slot]);
                    }
                    mbar_arrive(&ctl->full[slot]);
                }
            }
        }
        // drain: copies still in flight must land before the CTA exits
        cp_async_wait_all();
        if (lt == 0)
            for (int Lp = max(0, Lg - kStages); Lp < Lg; ++Lp) {
                volatile int never = 0;
                mbar_wait(&ctl->full[Lp % kStages], (Lp / kStages) & 1, &never, p.err);
            }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (+ Q loads)
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            const uint32_t id_qk_full = idesc_bf16(kRows, kBN, false, false);
            const uint32_t id_pv = idesc_bf16(kRows, kD, false, true);
            int q_issued = 0, q_done = 0;     // Q loads issued / waited for
            auto load_q = [&](int u) {
                ++q_issued;
                const Unit un = unit_of<PACKED>(p, u);
                mbar_arrive_expect_tx(&ctl->bar_q, 2 * kTileBytes);
                const int qrow = (u_tok0<PACKED>(p, un) + un.t0) * kH;
                for (int mt = 0; mt < 2; ++mt)
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d(sQ + mt * kTileBytes + h * kHalf, &tm_q, h * 64, qrow + mt * kRows,
                                    &ctl->bar_q);
            };
            int L0 = 0;                       // loads before this unit
            int J[2] = {0, 0};                // tiles before this unit, per M tile
            int k = 0;                        // units done
            bool ok = true;
            // nothing is loaded by a CTA that starts aborted
            if (blockIdx.x < n_units && !*abort) load_q(blockIdx.x);
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++k) {
                const Unit un = unit_of<PACKED>(p, u);
                const Geometry g = geometry<PACKED>(p, un);
                ok = q_issued > q_done && mbar_wait(&ctl->bar_q, k & 1, abort, p.err);
                if (ok) ++q_done;
                tc_fence_after();
                auto issue_qk = [&](int mt, int j) -> bool {
                    const TileRef r = tile_ref(p, g, mt, j);
                    const int ld = L0 + r.load;
                    const int slot = ld % kStages;
                    if (!mbar_wait(&ctl->full[slot], (ld / kStages) & 1, abort, p.err)) return false;
                    tc_fence_after();
                    // descriptors of the k-step 0 operands; a k step adds its byte
                    // offset / 16 to the start-address field (no carry: smem < 256 KB)
                    const uint64_t qd = sw128_desc(smem_u32(sQ + mt * kTileBytes), 16, 1024);
                    const uint64_t kd = sw128_desc(smem_u32(sK + slot * kTileBytes), 16, 1024);
                    const uint32_t idesc = (r.bn == kBN) ? id_qk_full : idesc_bf16(kRows, r.bn, false, false);
#pragma unroll
                    for (int kq = 0; kq < kD / 16; ++kq) {
                        const uint32_t off16 = ((kq >> 2) * kHalf + (kq & 3) * 32) >> 4;
                        mma_bf16_ss(tmem + mt * 128, qd + off16, kd + off16, idesc, kq > 0);
                    }
                    mma_commit(&ctl->s_full[mt]);
                    return true;
                };
                const int un_next = u + gridDim.x;
                // after the unit's last QK: once it has read Q, load the next unit's
                auto next_q = [&]() -> bool {
                    mma_commit(&ctl->q_free);
                    if (un_next >= n_units) return true;
                    if (!mbar_wait(&ctl->q_free, k & 1, abort, p.err) || *abort) return false;
                    load_q(un_next);
                    return true;
                };
                if (ok && g.T > 0) ok = issue_qk(0, 0) && issue_qk(1, 0);
                if (ok && g.T <= 1) ok = next_q();
                // the previous unit's O must have been read before this unit's first P.V
                bool o_ready[2] = {k == 0, k == 0};
                for (int j = 0; ok && j < g.T; ++j) {
                    for (int mt = 0; mt < 2 && ok; ++mt) {
                        if (!mbar_wait(&ctl->p_ready[mt], (J[mt] + j) & 1, abort, p.err)) { ok = false; break; }
                        if (!o_ready[mt]) {
                            if (!mbar_wait(&ctl->o_free[mt], (k - 1) & 1, abort, p.err)) { ok = false; break; }
                            o_ready[mt] = true;
                        }
                        tc_fence_after();
                        const TileRef r = tile_ref(p, g, mt, j);
                        const int ld = L0 + r.load;
                        const int slot = ld % kStages;
                        const uint64_t vd = sw128_desc(smem_u32(sK + slot * kTileBytes), kHalf, 1024);
                        // P sits in S (bf16, two per column): keys [32q, 32q+32)
                        // as hi weights in columns [32q, 32q+16) and lo weights in
                        // [32q+16, 32q+32); O += P_hi V + P_lo V per 16-key step
                        for (int kk = 0; kk < r.bn / 16; ++kk) {
                            const uint32_t pa = tmem + mt * 128 + (kk >> 1) * 32 + (kk & 1) * 8;
                            const uint64_t vk = vd + (uint64_t)(kk * (2048 >> 4));
                            mma_bf16_ts(tmem + 256 + mt * 128, pa, vk, id_pv, (j > 0 || kk > 0) ? 1u : 0u);
                            mma_bf16_ts(tmem + 256 + mt * 128, pa + 16, vk, id_pv, 1u);
                        }
                        if (r.last_consumer) mma_commit(&ctl->freeb[slot]);
                        if (j + 1 < g.T) {
                            ok = issue_qk(mt, j + 1);
                            if (ok && mt == 1 && j + 2 == g.T) ok = next_q();
                        }
                    }
                }
                // this unit's O is complete (or untouched when it has no tiles)
                if (ok) {
                    for (int mt = 0; mt < 2; ++mt) {
                        if (!o_ready[mt] && !mbar_wait(&ctl->o_free[mt], (k - 1) & 1, abort, p.err)) { ok = false; break; }
                        mma_commit(&ctl->o_full[mt]);
                    }
                }
                L0 += total_loads(p, g);
                J[0] += g.T;
                J[1] += g.T;
            }
            // every MMA issued must finish before TMEM is released, and a Q
            // load still in flight (the CTA aborted before waiting for it)
            // must land before the CTA's shared memory is given up
            mma_commit(&ctl->fin);
            volatile int never = 0;
            mbar_wait(&ctl->fin, 0, &never, p.err);
            if (q_issued > q_done) mbar_wait(&ctl->bar_q, q_done & 1, &never, p.err);
        }
        __syncwarp();
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------------ softmax
        const int mt = (warp - kSoftWarp0) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;                   // row of the M tile
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const int u_tok = r >> 6;                            // token of the M tile
        const uint32_t s_addr = tmem + lane_addr + mt * 128;
        const uint32_t o_addr = tmem + lane_addr + 256 + mt * 128;
        int J = 0;                                           // tiles before this unit
        int L0 = 0;                                          // loads before this unit
        int k = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++k) {
            const Unit un = unit_of<PACKED>(p, u);
            const int t0 = un.t0;
            const Geometry g = geometry<PACKED>(p, un);
            const int t = t0 + 2 * mt + u_tok;               // position in the sequence
            const bool row_ok = t < u_n<PACKED>(p, un);
            int Vt = 0;
            if (p.dense && row_ok) Vt = min((t + 1) / p.m, u_ne_dense<PACKED>(p, un));
            const int w_lo = t - p.window + 1;               // window [w_lo, t]
            // m_used: running max (base 2); l_r: sum of the bf16-rounded weights
            // (normalises O); l_e: sum of the unrounded weights (the lse output)
            float m_used = -INFINITY, l_r = 0.0f, l_e = 0.0f;
            for (int j = 0; j < g.T && ok; ++j) {
                const TileRef tr = tile_ref(p, g, mt, j);
                // every wait is warp-collective: the TMEM accesses below are .sync.aligned
                if (!__all_sync(0xffffffffu, mbar_wait(&ctl->s_full[mt], (J + j) & 1, abort, p.err))) { ok = false; break; }
                tc_fence_after();
                // which columns are keys of this row?
                int c_lo = 0, c_hi = -1;                     // contiguous range
                uint32_t mw[4] = {~0u, ~0u, ~0u, ~0u};       // gathered tiles: valid rows
                if (row_ok) {
                    if (tr.kind == 0) {
                        if (tr.token == u_tok) {
                            const int lg = L0 + tr.load;     // the loaders' index of this tile
                            const int slot = lg % kStages;
                            // the producer wrote the mask before arming this stage
                            if (!__all_sync(0xffffffffu, mbar_wait(&ctl->full[slot], (lg / kStages) & 1, abort, p.err))) { ok = false; break; }
#pragma unroll
                            for (int q = 0; q < 4; ++q) mw[q] = ctl->mask[slot][q];
                            c_hi = tr.bn - 1;
                        }
                    } else if (tr.kind == 1) {
                        c_hi = min(tr.bn, Vt - tr.chunk * kBN) - 1;
                    } else {
                        const int p0 = g.p_lo + tr.chunk * kBN;
                        c_lo = max(0, w_lo - p0);
                        c_hi = min(tr.bn, t - p0 + 1) - 1;
                    }
                }
                // (s_full of tile j is committed after the P.V of tile j-1 was issued
                // by the same thread, so that P.V has completed: O is stable and the
                // P columns are free)
                uint32_t vm[4];
                valid_bits(c_lo, c_hi, mw, vm);
                const bool has = (vm[0] | vm[1] | vm[2] | vm[3]) != 0u;
                float se = 0.0f, sr = 0.0f;
                if (!__any_sync(0xffffffffu, has)) {
                    // no key of this tile is visible to any row of the warp: P = 0
                    uint32_t zero[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) zero[i] = 0u;
#pragma unroll
                    for (int q = 0; q < 8; ++q) tmem_st16(s_addr + q * 16, zero);
                } else {
                    // pass 1: the tile's row max; raise the running max (and
                    // rescale O) when it grows by more than 2^8
                    const bool full = (vm[0] & vm[1] & vm[2] & vm[3]) == 0xffffffffu;   // uniform per warp
                    const float mx = full ? tile_max_full(s_addr, p.scale_log2) : tile_max(s_addr, vm, p.scale_log2);
                    const bool raise = mx > m_used + kRescaleLog2;   // true for a row's first keys
                    float alpha = 1.0f;
                    if (raise) {
                        alpha = (m_used == -INFINITY) ? 0.0f : ex2(m_used - mx);
                        m_used = mx;
                        l_r *= alpha;
                        l_e *= alpha;
                    }
                    if (j > 0 && __any_sync(0xffffffffu, raise)) rescale_o(o_addr, alpha);
                    // pass 2: P = exp2(z - m_used) over S
                    const float mm = (m_used == -INFINITY) ? INFINITY : m_used;
                    if (full)
                        tile_exp_full(s_addr, p.scale_log2, mm, p.lse != nullptr, se, sr);
                    else
                        tile_exp(s_addr, vm, p.scale_log2, mm, se, sr);
                    l_r += sr;
                    l_e += se;
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&ctl->p_ready[mt]);
            }
            if (!ok) break;
            // publish the row statistics of this unit for the epilogue
            stats[((k & 1) * 2 + mt) * kRows + r] = RowStat{m_used, l_r, l_e};
            mbar_arrive(&ctl->stats_ready[mt]);
            J += g.T;
            L0 += total_loads(p, g);
        }
    } else {
        // ------------------------------------------------------------ epilogue: O / l
        const int mt = (warp - kEpiWarp0) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const int u_tok = r >> 6;
        const uint32_t o_addr = tmem + lane_addr + 256 + mt * 128;
        int k = 0;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++k) {
            const Unit un = unit_of<PACKED>(p, u);
            const Geometry g = geometry<PACKED>(p, un);
            const int t = un.t0 + 2 * mt + u_tok;
            const bool row_ok = t < u_n<PACKED>(p, un);
            bool w_ok = mbar_wait(&ctl->stats_ready[mt], k & 1, abort, p.err);
            const RowStat st = stats[((k & 1) * 2 + mt) * kRows + r];
            w_ok = w_ok && mbar_wait(&ctl->o_full[mt], k & 1, abort, p.err);
            if (!__all_sync(0xffffffffu, w_ok)) break;
            tc_fence_after();
            __nv_bfloat16* orow = p.out + ((size_t)(u_tok0<PACKED>(p, un) + t) * kH + (r & 63)) * kD;
            if (g.T > 0) {
                const float inv = st.lr > 0.0f ? 1.0f / st.lr : 0.0f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float ov[32];
                    tmem_ld32(o_addr + q * 32, ov);
                    if (row_ok) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint4 v;
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(ov[i] * inv, ov[i + 1] * inv);
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(ov[i + 2] * inv, ov[i + 3] * inv);
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(ov[i + 4] * inv, ov[i + 5] * inv);
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(ov[i + 6] * inv, ov[i + 7] * inv);
                            v.x = *reinterpret_cast<uint32_t*>(&h0);
                            v.y = *reinterpret_cast<uint32_t*>(&h1);
                            v.z = *reinterpret_cast<uint32_t*>(&h2);
                            v.w = *reinterpret_cast<uint32_t*>(&h3);
                            *reinterpret_cast<uint4*>(orow + q * 32 + i) = v;
                        }
                    }
                }
                if (row_ok && p.lse)
                    p.lse[(size_t)(u_tok0<PACKED>(p, un) + t) * kH + (r & 63)] =
                        st.le > 0.0f ? (st.m + log2f(st.le)) / kLog2e : -INFINITY;
            } else if (row_ok) {
                // no key at all: o = 0, lse = -inf
                for (int i = 0; i < kD; i += 8) *reinterpret_cast<uint4*>(orow + i) = make_uint4(0, 0, 0, 0);
                if (p.lse) p.lse[(size_t)(u_tok0<PACKED>(p, un) + t) * kH + (r & 63)] = -INFINITY;
            }
            tc_fence_before();
            mbar_arrive(&ctl->o_free[mt]);
        }
    }

    // (the MMA issuer waited above for its final commit: no MMA is in flight)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------- host
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

// 2D bf16 tensor [rows, 128] with a 128-byte-swizzled box of {64, box_rows}.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool attention_tc_supported(const AttnArgs& a) {
    return a.dt == DT_BF16 && a.H == kH && a.D == kD && a.q_pos == nullptr &&
           a.raw_pos0 == nullptr && a.raw_len == nullptr && a.L_raw >= a.n_q && a.n_q > 0 &&
           a.topk <= 1024;   // the CTA's index rows are staged in shared memory
}

cudaError_t launch_attention_tc(const AttnArgs& a, uint32_t* err, cudaStream_t s) {
    CUtensorMap tm_q, tm_c, tm_w;
    const uint64_t q_rows = (uint64_t)a.B * a.n_q * kH;
    const uint64_t c_rows = (uint64_t)a.B * (a.N_cap > 0 ? a.N_cap : 1);
    const uint64_t w_rows = (uint64_t)a.B * a.L_raw;
    const void* kvc = a.kv_c ? a.kv_c : a.kv_raw;   // any valid address if there are no entries
    if (!make_map(&tm_q, a.q, q_rows, 128) ||
        !make_map(&tm_c, kvc, a.N_cap > 0 ? c_rows : w_rows, a.dense ? 128 : 1) ||
        !make_map(&tm_w, a.kv_raw, w_rows, 128))
        return cudaErrorInvalidValue;
    TcParams p;
    p.kv_c = kvc;
    p.idx = a.idx;
    p.topk = a.dense ? 0 : a.topk;
    p.n_entries = a.n_entries;
    p.m = a.m;
    p.dense = a.dense;
    p.B = a.B;
    p.n = a.n_q;
    p.N_cap = a.N_cap;
    p.L_raw = a.L_raw;
    p.window = a.window;
    p.scale_log2 = a.scale * kLog2e;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.lse = a.lse_out;
    p.err = err;
    int units = a.B * ((a.n_q + kTokens - 1) / kTokens);
    if (a.vl) {                                     // packed: units per sequence
        p.vl = *a.vl;
        p.vl.uoff[0] = 0;
        for (int q = 0; q < p.vl.S; ++q)
            p.vl.uoff[q + 1] = p.vl.uoff[q] + (p.vl.tok[q + 1] - p.vl.tok[q] + kTokens - 1) / kTokens;
        units = p.vl.uoff[p.vl.S];
        if (units == 0) return cudaSuccess;
    } else {
        p.vl.S = 0;
    }
    const size_t smem = kSmemFixed + (a.dense ? 0 : (size_t)kTokens * a.topk * sizeof(int));
    auto kern = a.vl ? attn_tc_kernel<true> : attn_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = units < sms ? units : sms;     // persistent: one CTA per SM
    kern<<<(unsigned)grid, kThreads, smem, s>>>(tm_q, tm_c, tm_w, p);
    count_launch();
    return cudaGetLastError();
}

}  // namespace csa
