// harp_quant_dev.cuh -- device helpers of the group quantizer shared by the
// kernels of libharp: PolarQuant (gist.science paper 2603.29078) section 2
// (RMS group scale to N(0,1), Lloyd-Max code, fp16 scale) and section 1
// (absmax uniform code), plus the LSB-first bit packing of the codes.
#pragma once

#include <cuda_fp16.h>

#include "harp_internal.h"

namespace harp {
namespace dq {

constexpr unsigned FULL = 0xffffffffu;

// Warp-wide reduction (xor butterfly, fixed order): sum or max.
__device__ __forceinline__ float warp_reduce(float v, bool is_max) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const float w = __shfl_xor_sync(FULL, v, o);
        v = is_max ? fmaxf(v, w) : v + w;
    }
    return v;
}

// Group scale from the combined statistic: RMS (sum of squares; Lloyd-Max's
// default) or max|x| / scale_div (absmax: qmax; Lloyd-Max's absmax mode: the
// largest centroid), rounded to fp16 (nearest even), saturating at 65504.
__device__ __forceinline__ unsigned short group_scale_bits(float stat, const QuantDev &Q) {
    float s;
    if (!Q.stat_max) {
        s = sqrtf(stat / static_cast<float>(Q.group));
    } else {
        s = stat / Q.scale_div;
    }
    s = fminf(s, 65504.0f);
    return __half_as_ushort(__float2half_rn(s));
}


// ------------------------------------------------------------ codes

// t[OFF + STRIDE * idx] for idx in [0, N) (N a power of two) by a tree of
// selects on the bits of idx: the array stays in registers.
template <int OFF, int N, int STRIDE, int K>
__device__ __forceinline__ float pick(const float (&t)[K], int idx) {
    if constexpr (N == 1) {
        return t[OFF];
    } else {
        return (idx & (N / 2)) ? pick<OFF + STRIDE * (N / 2), N / 2, STRIDE, K>(t, idx)
                               : pick<OFF, N / 2, STRIDE, K>(t, idx);
    }
}

// Lloyd-Max code = number of midpoints below z: binary search over the
// sorted fp32 midpoints held in registers (ties go to the lower code).
template <int BITS, int STEP = (1 << (BITS - 1))>
__device__ __forceinline__ int lm_search(float z, const float (&t)[(1 << BITS) - 1], int code) {
    if constexpr (STEP == 0) {
        return code;
    } else {
        constexpr int K = 1 << BITS;
        const float th = pick<STEP - 1, K / (2 * STEP), 2 * STEP, K - 1>(t, code / (2 * STEP));
        return lm_search<BITS, STEP / 2>(z, t, code + ((z > th) ? STEP : 0));
    }
}

template <int BITS>
__device__ __forceinline__ int code_of(float x, float s, float inv_s, bool lloyd,
                                       const float (&t)[(1 << BITS) - 1]) {
    constexpr int HALF = 1 << (BITS - 1);
    if (!(s > 0.0f)) return HALF;
    const float z = x * inv_s;
    if (lloyd) return lm_search<BITS>(z, t, 0);
    const float qmax = static_cast<float>(HALF - 1);
    return static_cast<int>(fminf(fmaxf(rintf(z), -qmax), qmax)) + HALF;
}

// The same code with the midpoints in shared memory (ts[k], k < 2^BITS - 1):
// a binary search of BITS dependent steps, each one load and one compare.
template <int BITS>
__device__ __forceinline__ int code_of_smem(float x, float s, float inv_s, bool lloyd, const float *ts) {
    constexpr int HALF = 1 << (BITS - 1);
    if (!(s > 0.0f)) return HALF;
    const float z = x * inv_s;
    if (lloyd) {
        int code = 0;
#pragma unroll
        for (int step = HALF; step >= 1; step >>= 1) code += (z > ts[code + step - 1]) ? step : 0;
        return code;
    }
    const float qmax = static_cast<float>(HALF - 1);
    return static_cast<int>(fminf(fmaxf(rintf(z), -qmax), qmax)) + HALF;
}

// Lloyd-Max code = number of midpoints below z by one table read and one
// compare: NB bins of width 8/NB over [-4, 4]; bin = rint(z * NB/8 + NB/2)
// clamped to [0, NB - 1] (one rounding of an exact product-sum, so z lies in
// [(bin - NB/2 - 1/2) * 8/NB, (bin - NB/2 + 1/2) * 8/NB] unless clamped);
// bins[bin] = number of midpoints below that lower edge (0 for bin 0). Exact
// when no bin holds two midpoints (bins_exact on the host); thr[K - 1] must
// be +inf.
template <int NB>
__device__ __forceinline__ int code_binned(float z, const float *thr, const unsigned char *bins) {
    const float y = fmaf(z, static_cast<float>(NB / 8), static_cast<float>(NB / 2) + 12582912.0f);  // 1.5 * 2^23
    int bin = __float_as_int(y) - 0x4B400000;
    bin = min(max(bin, 0), NB - 1);
    const int c = bins[bin];
    return c + ((z > thr[c]) ? 1 : 0);
}

// Entry i of that table, for thread i < NB (K - 1 midpoints in thr).
template <int NB>
__device__ __forceinline__ unsigned char bin_entry(int i, const float *thr, int K) {
    if (i == 0) return 0;
    const float lo = (static_cast<float>(i - NB / 2) - 0.5f) * (8.0f / NB);
    int c = 0;
    for (int k = 0; k < K - 1; ++k) c += (thr[k] < lo) ? 1 : 0;
    return static_cast<unsigned char>(c);
}

template <int BITS>
__device__ __forceinline__ unsigned pack_words(int code, int lane) {
    const int bit0 = BITS * lane;
    const int wlo = bit0 >> 5, sh = bit0 & 31;
    const unsigned lo = static_cast<unsigned>(code) << sh;
    const unsigned hi = (sh + BITS > 32) ? (static_cast<unsigned>(code) >> (32 - sh)) : 0u;
    unsigned mine = 0;
#pragma unroll
    for (int w = 0; w < BITS; ++w) {
        const unsigned part = (w == wlo ? lo : 0u) | (w == wlo + 1 ? hi : 0u);
        const unsigned word = __reduce_or_sync(FULL, part);
        if (w == lane) mine = word;
    }
    return mine;
}

// Group statistic of `g` consecutive values for one vector: each lane
// accumulates its values (coordinates lane, lane+32, ...) in order, then a
// fixed xor tree combines the lanes. The standalone quantizer uses the same
// order, so both give identical scales.
__device__ __forceinline__ float combine(float a, float x, bool is_max) {
    return is_max ? fmaxf(a, fabsf(x)) : fmaf(x, x, a);
}


}  // namespace dq
}  // namespace harp
