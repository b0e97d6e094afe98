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
//     and loaded once per CTA;
//   - sparse-mode compressed tiles belong to one token: their rows are
//     gathered by index, and the rows of the other token in the M tile are
//     masked.
// Arithmetic is fp16 on the tensor cores with fp32 accumulation: the loader
// warps read the bf16 key rows with 16-byte loads and write them converted
// to fp16 into the 128-byte-swizzled layout the tensor core reads; Q is
// converted in shared memory once per unit.  The conversion is exact for
// magnitudes in [2^-14, 65504] (smaller values keep an absolute error below
// 2^-25, larger ones saturate at 65504).  fp16 gives the softmax weights P
// 11 significant bits: a bf16 P (8 bits) moves the output by up to 2^-8 of
// the spread of the values it averages, several 1e-2 for keys of magnitude
// ~16.
// Roles (21 warps): warps 0-3 load (index rows, key tiles, the Q
// conversion); warp 4 allocates TMEM, loads each unit's Q by TMA and one
// lane issues every MMA; warps 5-12 and 13-20 run the softmax of M tile 0
// / 1: each row of an M tile belongs to two threads, one per 64-column half
// of the key tile (a warp reaches TMEM lanes 32*(warp%4) .. +31), which
// exchange their half-row maxima through shared memory once per tile; at
// the end of a unit the same threads normalise O and write their half of
// each output row.
// TMEM: S0 [cols 0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// S = Q K^T (M=128, N<=128, K=128 in 8 steps), P = exp2(S*scale*log2e - m)
// in fp16 written back into S (keys [32q, 32q+32) into columns [32q, 32q+16)),
// O += P V with P read from tensor memory and V the same shared tile read as
// an MN-major operand.  The running sum adds the fp16-rounded weights the MMA
// actually multiplies, so the result is an exact convex combination of the
// keys under those weights.  The running max is only raised (and O rescaled
// in TMEM) when it grows by more than 2^8, so most tiles need no rescale;
// the final division by the running sum is exact.
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
constexpr int kLoadWarps = 4;                      // loaders: index rows, key tiles, Q conversion
constexpr int kLoadThreads = kLoadWarps * 32;
constexpr int kMmaWarp = kLoadWarps;               // TMEM allocation, MMA issue, Q loads
constexpr int kSoftLo0 = kLoadWarps + 1;           // 4 + 4 warps: columns 0-63 of M tiles 0 / 1
constexpr int kSoftHi0 = kSoftLo0 + 8;             // 4 + 4 warps: columns 64-127 of M tiles 0 / 1
constexpr int kSoftWarps = 16;
constexpr int kThreads = (kLoadWarps + 1 + kSoftWarps) * 32;
static_assert(kLoadThreads == 128, "loaders cover the 128 rows of a tile, 16 lanes per row");
constexpr int kHalf = 16384;        // one 64-column half of a 128-row tile
constexpr int kTileBytes = 32768;   // 128 rows x 128 fp16
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;

struct __align__(8) Ctrl {
    uint64_t bar_q;                 // the unit's Q (bf16) has landed
    uint64_t q_conv;                // ... and is converted to fp16
    uint64_t q_free;                // the unit's last QK has read Q
    uint64_t o_full[2];             // the unit's last P.V has landed in O
    uint64_t o_free[2];             // the unit's output has been read out of O
    uint64_t full[kStages];
    uint64_t freeb[kStages];
    uint64_t s_full[2];
    uint64_t p_ready[2];
    uint64_t fin;
    uint64_t stall_bar;             // test hook: a barrier nothing completes
    uint64_t xbar[2][4];            // [M tile][quarter]: the two half-row warps meet
    uint32_t mask[kStages][4];      // gathered tiles: valid rows of the stage
    uint32_t tmem_base;
    int abort;
    int load_go[2];            // loaders: continue with the next load (alternating slots:
                               // decision d+1 is written only after every loader passed
                               // the barrier of decision d, so d is never overwritten
                               // before it is read)
};

// Exchange between the two half-row threads of a row (double-buffered by
// tile and by unit parity).
struct Xchg {
    float mx[2][2][2][kRows];       // [tile parity][M tile][half][row]: half-row maximum of S
    float l[2][2][2][2][kRows];     // [unit parity][M tile][half][rounded / exact][row]: partial sums
};
constexpr size_t kSmemFixed = 1024 /*align slack*/ + 2 * kTileBytes /*Q*/ +
                              kStages * kTileBytes + sizeof(Ctrl) + sizeof(Xchg);
// + the CTA's index rows (sparse mode): kTokens * topk int32

struct TcParams {
    const void* kv_c;          // [rows_c, 128] bf16: compressed entries (gathered or a dense prefix)
    const void* kv_raw;        // [rows_w, 128] bf16: raw rows (the window)
    const void* q;             // [B * n * 64, 128] bf16 (Q tiles also come by TMA)
    long rows_c, rows_w;       // rows present in memory (loads beyond them read zeros)
    const int* idx;            // sparse: [B, n, topk]
    int topk;
    const int* n_entries;      // dense
    int m;
    int dense;
    int B, n, N_cap, L_raw, window;
    int qpos0;                 // query q of every element sits at position qpos0 + q
    int rawpos0;               // raw row j of every element holds position rawpos0 + j
    float scale_log2;          // softmax scale * log2(e)
    __nv_bfloat16* out;
    float* lse;
    uint32_t* err;
    uint64_t wait_ns;          // time limit of each wait of the work
    int stall;                 // test hook: one thread waits on stall_bar first
    VarlenMap vl;              // packed sequences (vl.S > 0)
};

__device__ __forceinline__ int round16(int v) { return (v + 15) & ~15; }

// 2^x with the MUFU instruction (ex2.approx of -inf is +0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// A bf16 pair as an fp16 pair (nearest; saturating at +-65504).
__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t w) {
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xffff0000u);
    uint32_t d;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
__device__ __forceinline__ uint4 bf8_to_h8(uint4 v) {
    return make_uint4(bf2_to_h2(v.x), bf2_to_h2(v.y), bf2_to_h2(v.z), bf2_to_h2(v.w));
}
// Two fp32 weights as an fp16 pair, and the pair's rounded values.
__device__ __forceinline__ uint32_t f2_to_h2(float lo, float hi, float& rlo, float& rhi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    __half2 h = *reinterpret_cast<__half2*>(&d);
    const float2 r = __half22float2(h);
    rlo = r.x;
    rhi = r.y;
    return d;
}

struct Geometry {
    int cc;        // sparse: chunks of 128 in a token's index row
    int Tc;        // compressed tiles per M tile
    int Tw;        // window tiles
    int T;         // tiles per M tile
    int bn_c_last; // N of the last compressed tile
    int bn_w_last;
    int p_lo;      // first window position (absolute)
    int Lw;
    int Vmax;      // dense: entries needed by the CTA's last token
};



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

// A unit's tokens t0 .. sit at positions qpos0 + t0 .. (packed sequences:
// qpos0 = rawpos0 = 0); its window reads the raw rows present, positions
// [rawpos0, rawpos0 + L_raw).
template <bool PACKED>
__device__ __forceinline__ Geometry geometry(const TcParams& p, const Unit& un) {
    Geometry g;
    const int t0 = un.t0 + p.qpos0;                                  // positions
    const int t_last = min(un.t0 + kTokens - 1, u_n<PACKED>(p, un) - 1) + p.qpos0;
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
        g.p_lo = max(max(0, p.rawpos0), t0 - p.window + 1);
        const int p_hi = min(t_last, p.rawpos0 + u_L_raw<PACKED>(p, un) - 1);
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


__device__ __forceinline__ float f2lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }

// Row max (of raw S: the scale is positive, so the same element) over the
// valid columns of this thread's 64-column half (S columns at s_half).
// full: every column of the half is a key of the row.
__device__ __forceinline__ float half_max(uint32_t s_half, const uint32_t vm[2], bool full) {
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll 1
    for (int q = 0; q < 2; ++q) {
        const uint32_t mq = q == 0 ? vm[0] : vm[1];
        if (!__any_sync(0xffffffffu, mq != 0u)) continue;    // no key in this chunk for the warp
        float sv[32];
        tmem_ld32(s_half + q * 32, sv);
        if (full) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                mx0 = max3(mx0, sv[i], sv[i + 1]);
                mx1 = max3(mx1, sv[i + 2], sv[i + 3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if ((mq >> i) & 1u) mx0 = fmaxf(mx0, sv[i]);
        }
    }
    return fmaxf(mx0, mx1);
}

// P = exp2(S*sl2 - m) for the valid columns (0 elsewhere) of this thread's
// half, as fp16 pairs written over S: the 32 keys of chunk q (S columns
// [32q, 32q+32) of the half) get their weights in the chunk's first 16
// columns, which it has just read.  Accumulates the sum of the rounded
// weights (sr, what the MMA multiplies) and, when wanted, of the exact ones
// (se, for the log-sum-exp).  m = +inf writes zeros.
__device__ __forceinline__ void half_exp(uint32_t s_half, const uint32_t vm[2], bool full, float sl2,
                                         float m, bool want_se, float& se, float& sr) {
    const uint64_t sl2x2 = f2_pack(sl2, sl2), negm = f2_pack(-m, -m);
    uint64_t accr = 0, acce = 0;      // (+0, +0)
#pragma unroll 1
    for (int q = 0; q < 2; ++q) {
        const uint32_t mq = q == 0 ? vm[0] : vm[1];
        uint32_t pk[16];
        if (!__any_sync(0xffffffffu, mq != 0u)) {
            // no key in this chunk for the warp: P = 0 without the exponentials
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
            tmem_st16(s_half + q * 32, pk);
            continue;
        }
        float sv[32];
        tmem_ld32(s_half + q * 32, sv);
        if (full) {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const uint64_t z = f2_fma(f2_pack(sv[e], sv[e + 1]), sl2x2, negm);
                const float p0 = ex2(f2lo(z)), p1 = ex2(f2hi(z));
                float r0, r1;
                pk[e >> 1] = f2_to_h2(p0, p1, r0, r1);
                accr = f2_add(accr, f2_pack(r0, r1));
                if (want_se) acce = f2_add(acce, f2_pack(p0, p1));
            }
        } else {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const float z0 = ((mq >> e) & 1u) ? fmaf(sv[e], sl2, -m) : -INFINITY;
                const float z1 = ((mq >> (e + 1)) & 1u) ? fmaf(sv[e + 1], sl2, -m) : -INFINITY;
                const float p0 = ex2(z0), p1 = ex2(z1);
                float r0, r1;
                pk[e >> 1] = f2_to_h2(p0, p1, r0, r1);
                accr = f2_add(accr, f2_pack(r0, r1));
                if (want_se) acce = f2_add(acce, f2_pack(p0, p1));
            }
        }
        tmem_st16(s_half + q * 32, pk);
    }
    sr += f2lo(accr) + f2hi(accr);
    se += f2lo(acce) + f2hi(acce);
}

// The row max rose by more than 2^8: rescale this thread's half of O.
__device__ __noinline__ void rescale_o_half(uint32_t o_half, float alpha) {
#pragma unroll 1
    for (int q = 0; q < 2; ++q) {
        float ov[32];
        tmem_ld32(o_half + q * 32, ov);
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] *= alpha;
        tmem_st32(o_half + q * 32, ov);
    }
    tmem_st_wait();
}

// A key tile by the loader threads: 128 rows of 256 bytes, 16 lanes per row
// (16 bytes each), 8 rows per round, 8 rounds of loads in flight before
// their converted values are stored into the 128-byte-swizzled fp16 layout.
// src_of(row) gives the row's global address, or nullptr for a zero row.
template <typename SrcOf>
__device__ __forceinline__ void load_tile_h(uint8_t* dst, int lt, SrcOf src_of) {
    const int c16 = lt & 15, half = c16 >> 3, cc = c16 & 7;
#pragma unroll 1
    for (int it0 = 0; it0 < kBN / 8; it0 += 8) {
        uint4 v[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int row = (it0 + b) * 8 + (lt >> 4);
            const uint8_t* src = src_of(row);
            v[b] = src ? __ldg(reinterpret_cast<const uint4*>(src) + c16) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int row = (it0 + b) * 8 + (lt >> 4);
            *reinterpret_cast<uint4*>(dst + half * kHalf + row * 128 + ((cc ^ (row & 7)) << 4)) = bf8_to_h8(v[b]);
        }
    }
}

// 21 warps sit on the SM's four 16,384-register partitions as 6 + 5 + 5 + 5,
// so a thread may hold at most 80 registers (6 x 32 x 80 = 15,360).
template <bool PACKED>
__global__ void __maxnreg__(80)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = base;                                  // [2][32 KB]
    uint8_t* sK = sQ + 2 * kTileBytes;                   // [kStages][32 KB]
    Ctrl* ctl = reinterpret_cast<Ctrl*>(sK + kStages * kTileBytes);
    Xchg* xc = reinterpret_cast<Xchg*>(ctl + 1);
    int* sIdx = reinterpret_cast<int*>(xc + 1);          // [kTokens][topk]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_units = PACKED ? p.vl.uoff[p.vl.S] : p.B * ((p.n + kTokens - 1) / kTokens);
    volatile int* abort = &ctl->abort;

    if (threadIdx.x == 0) {
        mbar_init(&ctl->bar_q, 1);
        mbar_init(&ctl->q_conv, kLoadThreads);
        mbar_init(&ctl->q_free, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl->full[s], kLoadThreads);
            mbar_init(&ctl->freeb[s], 1);
        }
        for (int i = 0; i < 8; ++i) mbar_init(&ctl->xbar[i >> 2][i & 3], 2);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->s_full[i], 1);
            mbar_init(&ctl->p_ready[i], 8);          // one arrival per softmax warp of the M tile
            mbar_init(&ctl->o_full[i], 1);
            mbar_init(&ctl->o_free[i], 8);
        }
        mbar_init(&ctl->fin, 1);
        mbar_init(&ctl->stall_bar, 1);
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

    if (warp < kLoadWarps) {
        // ------------------------------------------------------------ loaders
        const int lt = threadIdx.x;                          // 0 .. 127
        const uint8_t* kvc = static_cast<const uint8_t*>(p.kv_c);
        const uint8_t* kvr = static_cast<const uint8_t*>(p.kv_raw);
        int Lg = 0;                                          // loads issued by this CTA
        int dn = 0;                                          // go / stop decisions taken
        int k = 0;                                           // units done
        bool go = true;
        for (int u = blockIdx.x; u < n_units && go; u += gridDim.x, ++k) {
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
            const long ent0 = u_ent0<PACKED>(p, un);
            const long raw0 = u_raw0<PACKED>(p, un);
            const int un_n = u_n<PACKED>(p, un), un_N = u_N<PACKED>(p, un), un_L = u_L_raw<PACKED>(p, un);
            // Q is converted after the unit's first two loads (which need no Q)
            const int q_at = min(2, NL);
            for (int L = 0; L <= NL; ++L) {
                if (L == q_at) {
                    // the unit's Q (bf16, by TMA) has landed: convert it in place.
                    // One thread waits and decides for all loaders.
                    if (lt == 0) ctl->load_go[dn & 1] = mbar_wait(&ctl->bar_q, k & 1, abort, p.err, p.wait_ns) ? 1 : 0;
                    named_sync(1, kLoadThreads);
                    if (!ctl->load_go[dn++ & 1]) { go = false; break; }
#pragma unroll 1
                    for (int i0 = lt; i0 < 2 * kTileBytes / 16; i0 += 8 * kLoadThreads) {
                        uint4 v[8];
#pragma unroll
                        for (int b = 0; b < 8; ++b) v[b] = *reinterpret_cast<const uint4*>(sQ + (size_t)(i0 + b * kLoadThreads) * 16);
#pragma unroll
                        for (int b = 0; b < 8; ++b) *reinterpret_cast<uint4*>(sQ + (size_t)(i0 + b * kLoadThreads) * 16) = bf8_to_h8(v[b]);
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&ctl->q_conv);
                }
                if (L == NL) break;
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
                    const bool okw = use == 0 || mbar_wait(&ctl->freeb[slot], (use - 1) & 1, abort, p.err, p.wait_ns);
                    ctl->load_go[dn & 1] = (okw && !*abort) ? 1 : 0;
                }
                named_sync(1, kLoadThreads);
                if (!ctl->load_go[dn++ & 1]) { go = false; break; }
                if (kind == 0) {
                    const int* ir = sIdx + token * p.topk + chunk * kBN;
                    const int tpos = t0 + token;
                    // valid-row mask: loader thread lt checks row lt
                    {
                        const int c = chunk * kBN + lt;
                        const int sv = (c < p.topk) ? ir[lt] : -1;
                        const bool okr = tpos < un_n && sv >= 0 && sv < un_N;
                        const uint32_t bits = __ballot_sync(0xffffffffu, okr);
                        if (lane == 0) ctl->mask[slot][warp] = bits;
                    }
                    load_tile_h(dst, lt, [&](int row) -> const uint8_t* {
                        const int c = chunk * kBN + row;
                        const int sv = (c < p.topk) ? ir[row] : -1;
                        // masked rows are zero rows
                        return (tpos < un_n && sv >= 0 && sv < un_N) ? kvc + (size_t)(ent0 + sv) * (kD * 2) : nullptr;
                    });
                } else if (kind == 1) {
                    load_tile_h(dst, lt, [&](int row) -> const uint8_t* {
                        const long gr = ent0 + (long)chunk * kBN + row;
                        return gr < p.rows_c ? kvc + (size_t)gr * (kD * 2) : nullptr;
                    });
                } else {
                    load_tile_h(dst, lt, [&](int row) -> const uint8_t* {
                        const int jr = g.p_lo - p.rawpos0 + chunk * kBN + row;   // raw row
                        const long gr = raw0 + jr;
                        return (jr < un_L && gr < p.rows_w) ? kvr + (size_t)gr * (kD * 2) : nullptr;
                    });
                }
                // the tile (and, for a gathered one, the mask) is written:
                // visible to the tensor core once every loader has arrived
                fence_proxy_async_smem();
                mbar_arrive(&ctl->full[slot]);
                ++Lg;
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (+ Q loads)
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            const uint32_t id_qk_full = idesc_f16(kRows, kBN, false, false);
            const uint32_t id_pv = idesc_f16(kRows, kD, false, true);
            int q_issued = 0, q_done = 0;     // Q loads issued / converted Q waited for
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
            // test hook: a wait that runs out (nothing completes stall_bar)
            if (p.stall) mbar_wait(&ctl->stall_bar, 0, abort, p.err, p.wait_ns);
            // nothing is loaded by a CTA that starts aborted
            if (blockIdx.x < n_units && !*abort) load_q(blockIdx.x);
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++k) {
                const Unit un = unit_of<PACKED>(p, u);
                const Geometry g = geometry<PACKED>(p, un);
                ok = q_issued > q_done && mbar_wait(&ctl->q_conv, k & 1, abort, p.err, p.wait_ns);
                if (ok) ++q_done;
                tc_fence_after();
                auto issue_qk = [&](int mt, int j) -> bool {
                    const TileRef r = tile_ref(p, g, mt, j);
                    const int ld = L0 + r.load;
                    const int slot = ld % kStages;
                    if (!mbar_wait(&ctl->full[slot], (ld / kStages) & 1, abort, p.err, p.wait_ns)) return false;
                    tc_fence_after();
                    // descriptors of the k-step 0 operands; a k step adds its byte
                    // offset / 16 to the start-address field (no carry: smem < 256 KB)
                    const uint64_t qd = sw128_desc(smem_u32(sQ + mt * kTileBytes), 16, 1024);
                    const uint64_t kd = sw128_desc(smem_u32(sK + slot * kTileBytes), 16, 1024);
                    const uint32_t idesc = (r.bn == kBN) ? id_qk_full : idesc_f16(kRows, r.bn, false, false);
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
                    if (!mbar_wait(&ctl->q_free, k & 1, abort, p.err, p.wait_ns) || *abort) return false;
                    load_q(un_next);
                    return true;
                };
                if (ok && g.T > 0) ok = issue_qk(0, 0) && issue_qk(1, 0);
                if (ok && g.T <= 1) ok = next_q();
                // the previous unit's O must have been read before this unit's first P.V
                bool o_ready[2] = {k == 0, k == 0};
                for (int j = 0; ok && j < g.T; ++j) {
                    for (int mt = 0; mt < 2 && ok; ++mt) {
                        if (!mbar_wait(&ctl->p_ready[mt], (J[mt] + j) & 1, abort, p.err, p.wait_ns)) { ok = false; break; }
                        if (!o_ready[mt]) {
                            if (!mbar_wait(&ctl->o_free[mt], (k - 1) & 1, abort, p.err, p.wait_ns)) { ok = false; break; }
                            o_ready[mt] = true;
                        }
                        tc_fence_after();
                        const TileRef r = tile_ref(p, g, mt, j);
                        const int ld = L0 + r.load;
                        const int slot = ld % kStages;
                        const uint64_t vd = sw128_desc(smem_u32(sK + slot * kTileBytes), kHalf, 1024);
                        // P sits in S (fp16, two per column): keys [32q, 32q+32) in
                        // columns [32q, 32q+16); one 16-key step per MMA
                        for (int kk = 0; kk < r.bn / 16; ++kk)
                            mma_bf16_ts(tmem + 256 + mt * 128, tmem + mt * 128 + (kk >> 1) * 32 + (kk & 1) * 8,
                                       vd + (uint64_t)(kk * (2048 >> 4)), id_pv, (j > 0 || kk > 0) ? 1u : 0u);
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
                        if (!o_ready[mt] && !mbar_wait(&ctl->o_free[mt], (k - 1) & 1, abort, p.err, p.wait_ns)) { ok = false; break; }
                        mma_commit(&ctl->o_full[mt]);
                    }
                }
                L0 += total_loads(p, g);
                J[0] += g.T;
                J[1] += g.T;
            }
            // every MMA issued must finish before TMEM is released, and a Q
            // load still in flight (the CTA aborted before it was converted)
            // must land before the CTA's shared memory is given up
            mma_commit(&ctl->fin);
            volatile int never = 0;
            mbar_wait(&ctl->fin, 0, &never, p.err);
            if (q_issued > 0) mbar_wait(&ctl->bar_q, (q_issued - 1) & 1, &never, p.err);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + output
        const int h = warp >= kSoftHi0 ? 1 : 0;               // which 64-column half of the tile
        const int mt = ((h ? warp - kSoftHi0 : warp - kSoftLo0) >> 2);
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;                   // row of the M tile
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const int u_tok = r >> 6;                            // token of the M tile
        const uint32_t s_half = tmem + lane_addr + mt * 128 + 64 * h;
        const uint32_t o_half = tmem + lane_addr + 256 + mt * 128 + 64 * h;
        // the row's two threads (two warps) meet on an mbarrier with bounded waits
        uint64_t* pair_bar = &ctl->xbar[mt][quarter];
        int xcount = 0;                                      // exchanges so far
        auto pair_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(pair_bar);
            const bool okx = __all_sync(0xffffffffu, mbar_wait(pair_bar, xcount & 1, abort, p.err, p.wait_ns));
            ++xcount;
            return okx;
        };
        int J = 0;                                           // tiles before this unit
        int L0 = 0;                                          // loads before this unit
        int k = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++k) {
            const Unit un = unit_of<PACKED>(p, u);
            const int t0 = un.t0;
            const Geometry g = geometry<PACKED>(p, un);
            const int t = t0 + 2 * mt + u_tok;               // the row's token
            const bool row_ok = t < u_n<PACKED>(p, un);
            const int tp = t + p.qpos0;                      // and its position
            int Vt = 0;
            if (p.dense && row_ok) Vt = min((tp + 1) / p.m, u_ne_dense<PACKED>(p, un));
            const int w_lo = tp - p.window + 1;              // window [w_lo, tp]
            // m_used: running max (base 2, shared by the row's two threads);
            // l_r / l_e: this half's sums of the rounded / exact weights
            float m_used = -INFINITY, l_r = 0.0f, l_e = 0.0f;
            for (int j = 0; j < g.T && ok; ++j) {
                const TileRef tr = tile_ref(p, g, mt, j);
                // every wait is warp-collective: the TMEM accesses below are .sync.aligned
                if (!__all_sync(0xffffffffu, mbar_wait(&ctl->s_full[mt], (J + j) & 1, abort, p.err, p.wait_ns))) { ok = false; break; }
                tc_fence_after();
                // which columns are keys of this row?
                int c_lo = 0, c_hi = -1;                     // contiguous range
                uint32_t mw[4] = {~0u, ~0u, ~0u, ~0u};       // gathered tiles: valid rows
                if (row_ok) {
                    if (tr.kind == 0) {
                        if (tr.token == u_tok) {
                            const int lg = L0 + tr.load;     // the loaders' index of this tile
                            const int slot = lg % kStages;
                            // the loaders wrote the mask before arriving on this stage
                            if (!__all_sync(0xffffffffu, mbar_wait(&ctl->full[slot], (lg / kStages) & 1, abort, p.err, p.wait_ns))) { ok = false; break; }
#pragma unroll
                            for (int q = 0; q < 4; ++q) mw[q] = ctl->mask[slot][q];
                            c_hi = tr.bn - 1;
                        }
                    } else if (tr.kind == 1) {
                        c_hi = min(tr.bn, Vt - tr.chunk * kBN) - 1;
                    } else {
                        const int p0 = g.p_lo + tr.chunk * kBN;
                        c_lo = max(0, w_lo - p0);
                        c_hi = min(tr.bn, tp - p0 + 1) - 1;
                    }
                }
                uint32_t vm4[4];
                valid_bits(c_lo, c_hi, mw, vm4);
                const uint32_t vm[2] = {h ? vm4[2] : vm4[0], h ? vm4[3] : vm4[1]};
                const bool has = (vm[0] | vm[1]) != 0u;
                const bool full = (vm[0] & vm[1]) == 0xffffffffu;
                const bool warp_has = __any_sync(0xffffffffu, has);
                // pass 1: this half's max; the row's max from both halves
                float hm = -INFINITY;
                if (warp_has) hm = half_max(s_half, vm, full);
                const int par = (J + j) & 1;
                xc->mx[par][mt][h][r] = hm;
                if (!pair_sync()) { ok = false; break; }
                const float tmx = fmaxf(hm, xc->mx[par][mt][h ^ 1][r]);
                // raise the running max (and rescale O) when it grows by more
                // than 2^8; both threads of the row decide alike
                bool raise = false;
                float alpha = 1.0f;
                if (tmx > -INFINITY) {
                    const float mx = tmx * p.scale_log2;
                    raise = mx > m_used + kRescaleLog2;      // true for a row's first keys
                    if (raise) {
                        alpha = (m_used == -INFINITY) ? 0.0f : ex2(m_used - mx);
                        m_used = mx;
                        l_r *= alpha;
                        l_e *= alpha;
                    }
                }
                if (j > 0 && __any_sync(0xffffffffu, raise)) rescale_o_half(o_half, alpha);
                // pass 2: P = exp2(z - m_used) over this half of S
                // (s_full of tile j is committed after the P.V of tile j-1 was issued
                // by the same thread, so that P.V has completed: O is stable and the
                // P columns are free)
                if (warp_has) {
                    const float mm = (m_used == -INFINITY) ? INFINITY : m_used;
                    float se = 0.0f, sr = 0.0f;
                    half_exp(s_half, vm, full, p.scale_log2, mm, p.lse != nullptr, se, sr);
                    l_r += sr;
                    l_e += se;
                } else {
                    // no key of this half is visible to any row of the warp: P = 0
                    uint32_t zero[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) zero[i] = 0u;
                    tmem_st16(s_half, zero);
                    tmem_st16(s_half + 32, zero);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->p_ready[mt]);
            }
            if (!ok) break;
            // ---------------------------------------------------------- unit end
            // the row's sums from both halves, then O / l for this half's 64 dims
            const int up = k & 1;
            xc->l[up][mt][h][0][r] = l_r;
            xc->l[up][mt][h][1][r] = l_e;
            if (!pair_sync()) break;
            const float LR = l_r + xc->l[up][mt][h ^ 1][0][r];
            const float LE = l_e + xc->l[up][mt][h ^ 1][1][r];
            if (!__all_sync(0xffffffffu, mbar_wait(&ctl->o_full[mt], k & 1, abort, p.err, p.wait_ns))) break;
            tc_fence_after();
            __nv_bfloat16* orow = p.out + ((size_t)(u_tok0<PACKED>(p, un) + t) * kH + (r & 63)) * kD + 64 * h;
            if (g.T > 0) {
                const float inv = LR > 0.0f ? 1.0f / LR : 0.0f;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    float ov[32];
                    tmem_ld32(o_half + q * 32, ov);
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
                if (row_ok && p.lse && h == 0)
                    p.lse[(size_t)(u_tok0<PACKED>(p, un) + t) * kH + (r & 63)] =
                        LE > 0.0f ? (m_used + log2f(LE)) / kLog2e : -INFINITY;
            } else if (row_ok) {
                // no key at all: o = 0, lse = -inf
                for (int i = 0; i < 64; i += 8) *reinterpret_cast<uint4*>(orow + i) = make_uint4(0, 0, 0, 0);
                if (p.lse && h == 0) p.lse[(size_t)(u_tok0<PACKED>(p, un) + t) * kH + (r & 63)] = -INFINITY;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->o_free[mt]);
            J += g.T;
            L0 += total_loads(p, g);
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
    // positions come as the uniform offsets pos0 / raw_base (per-element
    // arrays go to the row kernels)
    return a.dt == DT_BF16 && a.H == kH && a.D == kD && a.q_pos == nullptr &&
           a.raw_pos0 == nullptr && a.raw_len == nullptr && a.L_raw >= a.n_q && a.n_q > 0 &&
           a.topk <= 1024;   // the CTA's index rows are staged in shared memory
}

cudaError_t launch_attention_tc(const AttnArgs& a, uint32_t* err, cudaStream_t s) {
    CUtensorMap tm_q;
    const uint64_t q_rows = (uint64_t)a.B * a.n_q * kH;
    const uint64_t c_rows = (uint64_t)a.B * (a.N_cap > 0 ? a.N_cap : 0);
    const uint64_t w_rows = (uint64_t)a.B * a.L_raw;
    if (!make_map(&tm_q, a.q, q_rows, 128)) return cudaErrorInvalidValue;
    TcParams p;
    p.kv_c = a.kv_c ? a.kv_c : a.kv_raw;   // any valid address when there are no entries
    p.kv_raw = a.kv_raw;
    p.rows_c = a.kv_c ? (long)c_rows : 0;
    p.rows_w = (long)w_rows;
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
    p.qpos0 = a.vl ? 0 : a.pos0;
    p.rawpos0 = a.vl ? 0 : a.raw_base;
    p.scale_log2 = a.scale * kLog2e;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.lse = a.lse_out;
    p.err = err;
    p.wait_ns = wait_limit_ns();
    p.stall = take_stall();
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
    kern<<<(unsigned)grid, kThreads, smem, s>>>(tm_q, p);
    count_launch();
    return cudaGetLastError();
}

}  // namespace csa
