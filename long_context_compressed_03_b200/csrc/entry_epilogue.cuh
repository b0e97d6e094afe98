// entry_epilogue.cuh -- the store of compressed entries (stage 1), shared by
// the mean-pool and the gated compressors.
//
// rows[e][0 .. d_out) (fp32, shared memory) are written as entry row0 + e of
// the output: fp32 / bf16 stores, or one E4M3 row with scale = amax/448
// (1 for a zero row), code = E4M3(v / scale) by IEEE division, nearest even,
// saturating -- after a Walsh-Hadamard rotation of the row for the rotated
// type.  Every thread of the CTA calls it; warps take rows in turn.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace csa {

template <int OUT, int kThreads>
__device__ __forceinline__ void store_entry_rows(float* rows, int ne, int d_out, void* out_v,
                                                 float* row_scale, size_t row0, float hnorm) {
    const int tid = threadIdx.x;
    if constexpr (OUT == DT_E4M3 || OUT == DT_E4M3H) {
        const int warp = tid >> 5, lane = tid & 31;
        uint8_t* out = static_cast<uint8_t*>(out_v);
        for (int e = warp; e < ne; e += kThreads / 32) {
            if constexpr (OUT == DT_E4M3H) hadamard_row_warp(rows + e * d_out, d_out, hnorm);
            float amax = 0.0f;
            for (int o = lane; o < d_out; o += 32) amax = fmaxf(amax, fabsf(rows[e * d_out + o]));
            for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
            for (int o = lane; o < d_out; o += 32)
                out[(row0 + e) * d_out + o] = e4m3_code(__fdiv_rn(rows[e * d_out + o], scale));
            if (lane == 0) row_scale[row0 + e] = scale;
        }
    } else {
        using Tout = typename std::conditional<OUT == DT_F32, float, __nv_bfloat16>::type;
        Tout* out = static_cast<Tout*>(out_v) + row0 * d_out;
        constexpr int kV = 16 / (int)sizeof(Tout);          // values per 16-byte store
        if (d_out % kV == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0 &&
            (reinterpret_cast<uintptr_t>(rows) & 15u) == 0) {
            // the rows are contiguous in the output: 16-byte stores, same rounding
            const int nv = ne * d_out / kV;
            for (int p = tid; p < nv; p += kThreads) {
                const float4* r = reinterpret_cast<const float4*>(rows + p * kV);
                uint4 v;
                if constexpr (OUT == DT_F32) {
                    const float4 f = r[0];
                    v = make_uint4(__float_as_uint(f.x), __float_as_uint(f.y), __float_as_uint(f.z),
                                   __float_as_uint(f.w));
                } else {
                    const float4 f0 = r[0], f1 = r[1];
                    const __nv_bfloat162 h0 = __floats2bfloat162_rn(f0.x, f0.y);
                    const __nv_bfloat162 h1 = __floats2bfloat162_rn(f0.z, f0.w);
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(f1.x, f1.y);
                    const __nv_bfloat162 h3 = __floats2bfloat162_rn(f1.z, f1.w);
                    v = make_uint4(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1),
                                   *reinterpret_cast<const uint32_t*>(&h2), *reinterpret_cast<const uint32_t*>(&h3));
                }
                *reinterpret_cast<uint4*>(out + (size_t)p * kV) = v;
            }
        } else {
            for (int p = tid; p < ne * d_out; p += kThreads) store_out<Tout>(out + p, rows[p]);
        }
    }
}

}  // namespace csa
