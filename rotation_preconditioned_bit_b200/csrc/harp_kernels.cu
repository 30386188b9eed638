// harp_kernels.cu -- sm_100a kernels of libharp.
//
// What they compute:
//  * HARP (gist.science paper 2605.29843) section 2.1: a processor is a product
//    of stride stages; stage t applies a b_t x b_t block to every group of
//    coordinates {h b s + k s + l : k < b} (s = product of the later radices),
//    one block per group. Section 5: the inverse applies the transposes in
//    reverse order.
//  * PolarQuant (gist.science paper 2603.29078) section 2: group scale to
//    N(0,1) (RMS), Lloyd-Max code, fp16 scale; section 1: absmax uniform code.
//
// Design (B200): one CTA owns a tile of R whole vectors in shared memory as
// fp32, laid out [coordinate][vector] so that a lane reads the same
// coordinate of BT vectors with one vector load. Every stage is a batch of
// small GEMMs (per group: [b x b] block times [b x R] slice); a lane computes
// 4 outputs x BT vectors with FFMA, reading its 4 block coefficients with one
// 16-byte L1-cached load (the plan stores blocks padded and pre-transposed
// for this). Groups are processed in rounds of whole groups: compute into
// registers, barrier, write in place. The last stage of the forward row pass
// is followed, in the same kernel, by the group scale, the code search and
// LSB-first bit packing with warp-wide OR reductions.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "harp_internal.h"

namespace harp {
namespace {

constexpr int NT = 512;              // threads per CTA
constexpr int SMEM_MAX = 232448;     // opt-in dynamic shared memory per CTA (227 KB)
constexpr unsigned FULL = 0xffffffffu;

enum { SIDE_ROWS = 0, SIDE_COLS = 1 };

// ------------------------------------------------------------ small helpers

template <int BT>
__device__ __forceinline__ void lds(const float *p, float (&v)[BT]) {
    if constexpr (BT == 4) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else if constexpr (BT == 2) {
        const float2 t = *reinterpret_cast<const float2 *>(p);
        v[0] = t.x; v[1] = t.y;
    } else {
        v[0] = *p;
    }
}

template <int BT>
__device__ __forceinline__ void sts(float *p, const float (&v)[BT]) {
    if constexpr (BT == 4) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (BT == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    } else {
        *p = v[0];
    }
}

__device__ __forceinline__ float bf16_bits_to_float(unsigned short b) {
    return __uint_as_float(static_cast<unsigned>(b) << 16);
}

__device__ __forceinline__ unsigned short float_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Load 4 consecutive elements (16-byte f32 or 8-byte bf16 aligned).
template <int PRO>
__device__ __forceinline__ void ldg4(const void *base, int64_t off, float (&v)[4]) {
    if constexpr (PRO == PRO_F32) {
        const float4 t = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(base) + off));
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
        const uint2 t = __ldg(reinterpret_cast<const uint2 *>(
            static_cast<const unsigned short *>(base) + off));
        v[0] = __uint_as_float(t.x << 16);
        v[1] = __uint_as_float(t.x & 0xffff0000u);
        v[2] = __uint_as_float(t.y << 16);
        v[3] = __uint_as_float(t.y & 0xffff0000u);
    }
}

template <int PRO>
__device__ __forceinline__ float ldg1(const void *base, int64_t off) {
    if constexpr (PRO == PRO_F32) {
        return __ldg(static_cast<const float *>(base) + off);
    } else {
        return bf16_bits_to_float(__ldg(static_cast<const unsigned short *>(base) + off));
    }
}

template <int EPI>
__device__ __forceinline__ void stg4(void *base, int64_t off, const float (&v)[4]) {
    if constexpr (EPI == EPI_BF16) {
        uint2 t;
        t.x = float_to_bf16_bits(v[0]) | (static_cast<unsigned>(float_to_bf16_bits(v[1])) << 16);
        t.y = float_to_bf16_bits(v[2]) | (static_cast<unsigned>(float_to_bf16_bits(v[3])) << 16);
        *reinterpret_cast<uint2 *>(static_cast<unsigned short *>(base) + off) = t;
    } else {
        *reinterpret_cast<float4 *>(static_cast<float *>(base) + off) = make_float4(v[0], v[1], v[2], v[3]);
    }
}

template <int EPI>
__device__ __forceinline__ void stg1(void *base, int64_t off, float v) {
    if constexpr (EPI == EPI_BF16) {
        static_cast<unsigned short *>(base)[off] = float_to_bf16_bits(v);
    } else {
        static_cast<float *>(base)[off] = v;
    }
}

// Warp-wide reduction (xor butterfly, fixed order): sum or max.
__device__ __forceinline__ float warp_reduce(float v, bool is_max) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const float w = __shfl_xor_sync(FULL, v, o);
        v = is_max ? fmaxf(v, w) : v + w;
    }
    return v;
}

// Group scale from the combined statistic: RMS (Lloyd-Max) or absmax/qmax,
// rounded to fp16 (nearest even), saturating at 65504.
__device__ __forceinline__ unsigned short group_scale_bits(float stat, const QuantDev &Q) {
    float s;
    if (Q.kind == HARP_LLOYD_MAX) {
        s = sqrtf(stat / static_cast<float>(Q.group));
    } else {
        s = stat / static_cast<float>((1 << (Q.bits - 1)) - 1);
    }
    s = fminf(s, 65504.0f);
    return __half_as_ushort(__float2half_rn(s));
}

// Code of one value given its group's stored scale (as float) and the fp32
// midpoint table (Lloyd-Max: number of midpoints below x/s; absmax: rounded
// and clamped x/s, offset by 2^(b-1)). A zero scale gives the middle code.
__device__ __forceinline__ int quant_code(float x, float s, const QuantDev &Q, const float *thr) {
    const int half = 1 << (Q.bits - 1);
    if (!(s > 0.0f)) return half;
    const float z = x * __frcp_rn(s);
    if (Q.kind == HARP_LLOYD_MAX) {
        int code = 0;
        for (int step = half; step >= 1; step >>= 1)
            if (z > thr[code + step - 1]) code += step;
        return code;
    }
    const float qmax = static_cast<float>(half - 1);
    const float q = fminf(fmaxf(rintf(z), -qmax), qmax);
    return static_cast<int>(q) + half;
}

// Pack the warp's 32 consecutive codes (lane = position) into `bits` 32-bit
// words of the LSB-first bitstream; returns word `lane` (valid for lane < bits).
__device__ __forceinline__ unsigned pack_warp(int code, int bits, int lane) {
    const int bit0 = bits * lane;
    const int wlo = bit0 >> 5, sh = bit0 & 31;
    const unsigned lo = static_cast<unsigned>(code) << sh;
    const unsigned hi = (sh + bits > 32) ? (static_cast<unsigned>(code) >> (32 - sh)) : 0u;
    unsigned mine = 0;
    for (int w = 0; w < bits; ++w) {
        const unsigned part = (w == wlo ? lo : 0u) | (w == wlo + 1 ? hi : 0u);
        const unsigned word = __reduce_or_sync(FULL, part);
        if (w == lane) mine = word;
    }
    return mine;
}

// ------------------------------------------------------------ stage core

// One stride stage on the shared tile X[coord * Rp + vector] (R vectors).
// A unit is (group, 4 consecutive outputs, BT consecutive vectors); units of
// whole groups are handed out round by round.
template <int BT>
__device__ __forceinline__ void run_stage(float *X, int Rp, int R, int d, const StageDev &S,
                                          int dir, int tid) {
    constexpr int UPT = (BT == 4) ? 4 : 8;   // units per thread per round
    const int b = S.b, kpad = S.kpad, nk = kpad >> 2;
    const int s = static_cast<int>(S.s);
    const float *__restrict__ A = (dir == HARP_FWD) ? S.fwd : S.inv;
    const int nbq = R / BT;
    const int Ug = nk * nbq;          // units per group
    const int ngroups = d / b;
    int Gr = (UPT * NT) / Ug;         // whole groups per round
    if (Gr < 1) Gr = 1;
    const int sRp = s * Rp;

    for (int g0 = 0; g0 < ngroups; g0 += Gr) {
        const int gcount = min(Gr, ngroups - g0);
        const int nunits = gcount * Ug;
        float acc[UPT][4][BT];
        int aoff[UPT], xoff[UPT], sk[UPT];
#pragma unroll
        for (int u = 0; u < UPT; ++u) {
            const int unit = tid + u * NT;
            const int uu = (unit < nunits) ? unit : 0;
            const int q = uu / Ug;
            const int rem = uu - q * Ug;
            const int kq = rem / nbq;
            const int bq = rem - kq * nbq;
            const int c = g0 + q;
            const int h = c / s;
            const int l = c - h * s;
            aoff[u] = c * b * kpad + kq * 4;
            xoff[u] = (h * b * s + l) * Rp + bq * BT;
            sk[u] = q % b;           // skew the j order per group: spreads smem banks
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int v = 0; v < BT; ++v) acc[u][k][v] = 0.0f;
        }
#pragma unroll 1
        for (int jj = 0; jj < b; ++jj) {
#pragma unroll
            for (int u = 0; u < UPT; ++u) {
                int j = jj + sk[u];
                j -= (j >= b) ? b : 0;
                const float4 a = __ldg(reinterpret_cast<const float4 *>(A + aoff[u] + j * kpad));
                float x[BT];
                lds<BT>(X + xoff[u] + j * sRp, x);
#pragma unroll
                for (int v = 0; v < BT; ++v) {
                    acc[u][0][v] = fmaf(a.x, x[v], acc[u][0][v]);
                    acc[u][1][v] = fmaf(a.y, x[v], acc[u][1][v]);
                    acc[u][2][v] = fmaf(a.z, x[v], acc[u][2][v]);
                    acc[u][3][v] = fmaf(a.w, x[v], acc[u][3][v]);
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < UPT; ++u) {
            const int unit = tid + u * NT;
            if (unit < nunits) {
                const int kq4 = ((unit % Ug) / nbq) * 4;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (kq4 + k < b) sts<BT>(X + xoff[u] + (kq4 + k) * sRp, acc[u][k]);
            }
        }
    }
    __syncthreads();
}

// ------------------------------------------------------------ the kernel

template <int SIDE, int BT, int PRO, int EPI>
__global__ void __launch_bounds__(NT, 1)
vec_kernel(const PlanDev P, const QuantDev Q, const VecLaunch L, const int R) {
    extern __shared__ float4 smem_f4[];
    float *X = reinterpret_cast<float *>(smem_f4);
    const int tid = threadIdx.x;
    const int d = static_cast<int>(P.d);
    const int Rp = R;
    const int64_t v0 = static_cast<int64_t>(blockIdx.x) * R;
    const int64_t nvec = L.nvec;
    const bool fwd = (L.dir == HARP_FWD);
    const float *__restrict__ signs = P.signs;

    // ---------------------------------------------------------- prologue
    if constexpr (PRO == PRO_CODES) {
        // dequantise R rows of codes into the tile (inverse path)
        float *lev = X + static_cast<size_t>(d) * Rp;
        if (tid < 16) lev[tid] = Q.level[tid];
        __syncthreads();
        const int bits = Q.bits, g = Q.group, ng = d / g;
        const int64_t rowbytes = static_cast<int64_t>(d) * bits / 8;
        const unsigned mask = (1u << bits) - 1u;
        for (int idx = tid; idx < R * d; idx += NT) {
            const int r = idx / d, i = idx - r * d;
            const int64_t row = v0 + r;
            float val = 0.0f;
            if (row < nvec) {
                const int64_t bitoff = static_cast<int64_t>(i) * bits;
                const int64_t byte = bitoff >> 3;
                const uint8_t *cr = L.in_codes + row * rowbytes;
                unsigned w = cr[byte];
                if (byte + 1 < rowbytes) w |= static_cast<unsigned>(cr[byte + 1]) << 8;
                const int code = static_cast<int>((w >> (bitoff & 7)) & mask);
                const float s = __half2float(__ushort_as_half(L.in_scales[row * ng + i / g]));
                val = s * lev[code];
            }
            X[i * Rp + r] = val;
        }
    } else if constexpr (SIDE == SIDE_ROWS) {
        if ((R & 3) == 0 && (d & 3) == 0) {
            const int nc4 = d >> 2;
            for (int idx = tid; idx < (R >> 2) * nc4; idx += NT) {
                const int rq = idx / nc4, c4 = idx - rq * nc4;
                float v[4][4];
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const int64_t row = v0 + rq * 4 + rr;
                    if (row < nvec) {
                        ldg4<PRO>(L.in, row * L.ld_in + c4 * 4, v[rr]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) v[rr][e] = 0.0f;
                    }
                }
                if (fwd) {
                    const float4 sg = __ldg(reinterpret_cast<const float4 *>(signs) + c4);
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        v[rr][0] *= sg.x; v[rr][1] *= sg.y; v[rr][2] *= sg.z; v[rr][3] *= sg.w;
                    }
                }
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int e = (p + idx) & 3;
                    float w[4];
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        // select v[rr][e] without dynamic register indexing
                        w[rr] = (e == 0) ? v[rr][0] : (e == 1) ? v[rr][1] : (e == 2) ? v[rr][2] : v[rr][3];
                    }
                    *reinterpret_cast<float4 *>(X + (c4 * 4 + e) * Rp + rq * 4) =
                        make_float4(w[0], w[1], w[2], w[3]);
                }
            }
        } else {
            for (int idx = tid; idx < R * d; idx += NT) {
                const int r = idx / d, i = idx - r * d;
                const int64_t row = v0 + r;
                float val = (row < nvec) ? ldg1<PRO>(L.in, row * L.ld_in + i) : 0.0f;
                if (fwd) val *= __ldg(signs + i);
                X[i * Rp + r] = val;
            }
        }
    } else {  // SIDE_COLS: vectors are columns v0 .. v0+R-1, coordinates are rows
        if ((R & 3) == 0) {
            const int nq = R >> 2;
            for (int idx = tid; idx < d * nq; idx += NT) {
                const int i = idx / nq, bq = idx - i * nq;
                const int64_t col = v0 + bq * 4;
                float v[4];
                if (col + 3 < nvec) {
                    ldg4<PRO>(L.in, static_cast<int64_t>(i) * L.ld_in + col, v);
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        v[e] = (col + e < nvec) ? ldg1<PRO>(L.in, static_cast<int64_t>(i) * L.ld_in + col + e) : 0.0f;
                }
                if (fwd) {
                    const float sg = __ldg(signs + i);
#pragma unroll
                    for (int e = 0; e < 4; ++e) v[e] *= sg;
                }
                *reinterpret_cast<float4 *>(X + i * Rp + bq * 4) = make_float4(v[0], v[1], v[2], v[3]);
            }
        } else {
            for (int idx = tid; idx < d * R; idx += NT) {
                const int i = idx / R, bcol = idx - i * R;
                const int64_t col = v0 + bcol;
                float val = (col < nvec) ? ldg1<PRO>(L.in, static_cast<int64_t>(i) * L.ld_in + col) : 0.0f;
                if (fwd) val *= __ldg(signs + i);
                X[i * Rp + bcol] = val;
            }
        }
    }
    __syncthreads();

    // ---------------------------------------------------------- stages
    for (int ti = 0; ti < P.m; ++ti) {
        const int t = fwd ? ti : P.m - 1 - ti;
        run_stage<BT>(X, Rp, R, d, P.st[t], L.dir, tid);
    }

    // ---------------------------------------------------------- epilogue
    if constexpr (EPI == EPI_F32 || EPI == EPI_BF16) {
        if constexpr (SIDE == SIDE_ROWS) {
            if ((R & 3) == 0 && (d & 3) == 0) {
                const int nc4 = d >> 2;
                for (int idx = tid; idx < (R >> 2) * nc4; idx += NT) {
                    const int rq = idx / nc4, c4 = idx - rq * nc4;
                    float v[4][4];  // [row][e]
                    float sg[4] = {1.0f, 1.0f, 1.0f, 1.0f};
                    if (!fwd) {
                        const float4 t4 = __ldg(reinterpret_cast<const float4 *>(signs) + c4);
                        sg[0] = t4.x; sg[1] = t4.y; sg[2] = t4.z; sg[3] = t4.w;
                    }
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const int e = (p + idx) & 3;
                        const float4 w = *reinterpret_cast<const float4 *>(X + (c4 * 4 + e) * Rp + rq * 4);
                        const float se = (e == 0) ? sg[0] : (e == 1) ? sg[1] : (e == 2) ? sg[2] : sg[3];
#pragma unroll
                        for (int rr = 0; rr < 4; ++rr) {
                            const float val = ((rr == 0) ? w.x : (rr == 1) ? w.y : (rr == 2) ? w.z : w.w) * se;
                            if (e == 0) v[rr][0] = val;
                            else if (e == 1) v[rr][1] = val;
                            else if (e == 2) v[rr][2] = val;
                            else v[rr][3] = val;
                        }
                    }
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        const int64_t row = v0 + rq * 4 + rr;
                        if (row < nvec) stg4<EPI>(L.out, row * L.ld_out + c4 * 4, v[rr]);
                    }
                }
            } else {
                for (int idx = tid; idx < R * d; idx += NT) {
                    const int r = idx / d, i = idx - r * d;
                    const int64_t row = v0 + r;
                    float val = X[i * Rp + r];
                    if (!fwd) val *= __ldg(signs + i);
                    if (row < nvec) stg1<EPI>(L.out, row * L.ld_out + i, val);
                }
            }
        } else {  // SIDE_COLS
            if ((R & 3) == 0) {
                const int nq = R >> 2;
                for (int idx = tid; idx < d * nq; idx += NT) {
                    const int i = idx / nq, bq = idx - i * nq;
                    const int64_t col = v0 + bq * 4;
                    const float4 w = *reinterpret_cast<const float4 *>(X + i * Rp + bq * 4);
                    const float sg = fwd ? 1.0f : __ldg(signs + i);
                    float v[4] = {w.x * sg, w.y * sg, w.z * sg, w.w * sg};
                    if (col + 3 < nvec) {
                        stg4<EPI>(L.out, static_cast<int64_t>(i) * L.ld_out + col, v);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (col + e < nvec) stg1<EPI>(L.out, static_cast<int64_t>(i) * L.ld_out + col + e, v[e]);
                    }
                }
            } else {
                for (int idx = tid; idx < d * R; idx += NT) {
                    const int i = idx / R, bcol = idx - i * R;
                    const int64_t col = v0 + bcol;
                    float val = X[i * Rp + bcol];
                    if (!fwd) val *= __ldg(signs + i);
                    if (col < nvec) stg1<EPI>(L.out, static_cast<int64_t>(i) * L.ld_out + col, val);
                }
            }
        }
    } else {
        // EPI_QUANT / EPI_QUANT_F32: rows side, forward. g % 32 == 0, g | d.
        const int g = Q.group, ng = d / g, nchunk = d >> 5, cpg = g >> 5;
        float *part = X + static_cast<size_t>(d) * Rp;   // [R][nchunk]
        float *sc = part + R * nchunk;                    // [R][ng]
        float *thr = sc + R * ng;                         // [16]
        if (tid < 16) thr[tid] = Q.thr[tid];
        const bool is_max = (Q.kind == HARP_ABSMAX);
        const int warp = tid >> 5, lane = tid & 31;
        const int nrv = R / BT;
        // pass 1: per 32-coordinate chunk statistics
        for (int item = warp; item < nrv * nchunk; item += NT / 32) {
            const int rq = item / nchunk, ch = item - rq * nchunk;
            float x[BT];
            lds<BT>(X + (ch * 32 + lane) * Rp + rq * BT, x);
#pragma unroll
            for (int v = 0; v < BT; ++v) {
                const float st = warp_reduce(is_max ? fabsf(x[v]) : x[v] * x[v], is_max);
                if (lane == 0) part[(rq * BT + v) * nchunk + ch] = st;
            }
        }
        __syncthreads();
        // pass 2: group scales (combined in chunk order)
        for (int idx = tid; idx < R * ng; idx += NT) {
            const int r = idx / ng, gi = idx - r * ng;
            float stat = 0.0f;
            for (int c = 0; c < cpg; ++c) {
                const float p = part[r * nchunk + gi * cpg + c];
                stat = is_max ? fmaxf(stat, p) : stat + p;
            }
            const unsigned short hb = group_scale_bits(stat, Q);
            sc[idx] = __half2float(__ushort_as_half(hb));
            const int64_t row = v0 + r;
            if (row < nvec) L.scales[row * ng + gi] = hb;
        }
        __syncthreads();
        // pass 3: codes, packing (and the optional fp32 copy of the rotated rows)
        const int bits = Q.bits;
        const int64_t rowbytes = static_cast<int64_t>(d) * bits / 8;
        for (int item = warp; item < nrv * nchunk; item += NT / 32) {
            const int rq = item / nchunk, ch = item - rq * nchunk;
            const int i = ch * 32 + lane;
            const int gi = (ch * 32) / g;
            float x[BT];
            lds<BT>(X + i * Rp + rq * BT, x);
#pragma unroll
            for (int v = 0; v < BT; ++v) {
                const int r = rq * BT + v;
                const int64_t row = v0 + r;
                const int code = quant_code(x[v], sc[r * ng + gi], Q, thr);
                const unsigned word = pack_warp(code, bits, lane);
                if (row < nvec) {
                    if (lane < bits)
                        reinterpret_cast<unsigned *>(L.codes + row * rowbytes)[ch * bits + lane] = word;
                    if constexpr (EPI == EPI_QUANT_F32)
                        static_cast<float *>(L.out)[row * L.ld_out + i] = x[v];
                }
            }
        }
    }
}

// ------------------------------------------------------------ standalone codec

// One warp per (row, group): statistics chunk by chunk in the same order as
// the fused epilogue, then codes and packing.
template <int PRO>
__global__ void __launch_bounds__(256)
quantize_kernel(const QuantDev Q, const void *in, int64_t rows, int64_t cols, int64_t ld_in,
                uint8_t *codes, uint16_t *scales) {
    __shared__ float thr[16];
    if (threadIdx.x < 16) thr[threadIdx.x] = Q.thr[threadIdx.x];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int g = Q.group, bits = Q.bits;
    const int64_t ng = cols / g;
    const int64_t rowbytes = cols * bits / 8;
    const bool is_max = (Q.kind == HARP_ABSMAX);
    for (int64_t item = warp; item < rows * ng; item += nwarps) {
        const int64_t row = item / ng, gi = item - row * ng;
        const int64_t off = row * ld_in + gi * g;
        float stat = 0.0f;
        for (int c = 0; c < (g >> 5); ++c) {
            const float x = ldg1<PRO>(in, off + c * 32 + lane);
            const float p = warp_reduce(is_max ? fabsf(x) : x * x, is_max);
            stat = is_max ? fmaxf(stat, p) : stat + p;
        }
        const unsigned short hb = group_scale_bits(stat, Q);
        if (lane == 0) scales[row * ng + gi] = hb;
        const float s = __half2float(__ushort_as_half(hb));
        for (int c = 0; c < (g >> 5); ++c) {
            const float x = ldg1<PRO>(in, off + c * 32 + lane);
            const int code = quant_code(x, s, Q, thr);
            const unsigned word = pack_warp(code, bits, lane);
            if (lane < bits)
                reinterpret_cast<unsigned *>(codes + row * rowbytes)[((gi * g) >> 5) * bits + c * bits + lane] = word;
        }
    }
}

template <int EPI>
__global__ void __launch_bounds__(256)
dequantize_kernel(const QuantDev Q, const uint8_t *codes, const uint16_t *scales, int64_t rows,
                  int64_t cols, void *out, int64_t ld_out) {
    const int bits = Q.bits, g = Q.group;
    const int64_t ng = cols / g, rowbytes = cols * bits / 8;
    const unsigned mask = (1u << bits) - 1u;
    const int64_t n = rows * cols;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = idx / cols, i = idx - row * cols;
        const int64_t bitoff = i * bits, byte = bitoff >> 3;
        const uint8_t *cr = codes + row * rowbytes;
        unsigned w = cr[byte];
        if (byte + 1 < rowbytes) w |= static_cast<unsigned>(cr[byte + 1]) << 8;
        const int code = static_cast<int>((w >> (bitoff & 7)) & mask);
        const float s = __half2float(__ushort_as_half(scales[row * ng + i / g]));
        stg1<EPI>(out, row * ld_out + i, s * Q.level[code]);
    }
}

// ------------------------------------------------------------ host dispatch

int extra_smem_floats(int R, int d, int epi, int pro, int group) {
    int extra = 0;
    if (epi == EPI_QUANT || epi == EPI_QUANT_F32) extra += R * (d / 32) + R * (d / group) + 16;
    if (pro == PRO_CODES) extra += 16;
    return extra;
}

int pick_tile(int64_t d, int epi, int pro, int group) {
    static const int cand[] = {32, 28, 24, 20, 16, 12, 8, 6, 4, 2, 1};
    for (int R : cand) {
        const int64_t floats = d * R + extra_smem_floats(R, static_cast<int>(d), epi, pro, group);
        if (floats * 4 <= SMEM_MAX) return R;
    }
    return 0;
}

using KernelFn = void (*)(const PlanDev, const QuantDev, const VecLaunch, const int);

template <int SIDE, int BT, int PRO, int EPI>
KernelFn get_kernel() {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(vec_kernel<SIDE, BT, PRO, EPI>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_MAX);
    });
    return attr_err == cudaSuccess ? vec_kernel<SIDE, BT, PRO, EPI> : nullptr;
}

template <int SIDE, int BT>
KernelFn select_pe(int pro, int epi) {
    if constexpr (SIDE == SIDE_ROWS) {
        if (pro == PRO_CODES) {
            if (epi == EPI_F32) return get_kernel<SIDE, BT, PRO_CODES, EPI_F32>();
            if (epi == EPI_BF16) return get_kernel<SIDE, BT, PRO_CODES, EPI_BF16>();
            return nullptr;
        }
#define HARP_ROW_CASE(P)                                                          \
    if (pro == P) {                                                               \
        if (epi == EPI_F32) return get_kernel<SIDE, BT, P, EPI_F32>();            \
        if (epi == EPI_BF16) return get_kernel<SIDE, BT, P, EPI_BF16>();          \
        if (epi == EPI_QUANT) return get_kernel<SIDE, BT, P, EPI_QUANT>();        \
        if (epi == EPI_QUANT_F32) return get_kernel<SIDE, BT, P, EPI_QUANT_F32>(); \
    }
        HARP_ROW_CASE(PRO_F32)
        HARP_ROW_CASE(PRO_BF16)
#undef HARP_ROW_CASE
        return nullptr;
    } else {
        if (pro == PRO_F32 && epi == EPI_F32) return get_kernel<SIDE, BT, PRO_F32, EPI_F32>();
        if (pro == PRO_F32 && epi == EPI_BF16) return get_kernel<SIDE, BT, PRO_F32, EPI_BF16>();
        if (pro == PRO_BF16 && epi == EPI_F32) return get_kernel<SIDE, BT, PRO_BF16, EPI_F32>();
        if (pro == PRO_BF16 && epi == EPI_BF16) return get_kernel<SIDE, BT, PRO_BF16, EPI_BF16>();
        return nullptr;
    }
}

template <int SIDE>
KernelFn select_bt(int bt, int pro, int epi) {
    if (bt == 4) return select_pe<SIDE, 4>(pro, epi);
    if (bt == 2) return select_pe<SIDE, 2>(pro, epi);
    return select_pe<SIDE, 1>(pro, epi);
}

}  // namespace

int vec_tile(int64_t d, int epi, int group) {
    return pick_tile(d, epi, PRO_F32, group > 0 ? group : 32);
}

int launch_vec(const PlanDev &plan, const QuantDev *q, const VecLaunch &L, void *stream) {
    const int group = q ? q->group : 32;
    const int R = pick_tile(plan.d, L.epi, L.pro, group);
    if (R == 0) return static_cast<int>(cudaErrorInvalidValue);
    const int bt = (R % 4 == 0) ? 4 : (R % 2 == 0) ? 2 : 1;
    KernelFn fn = (L.side == HARP_RIGHT) ? select_bt<SIDE_ROWS>(bt, L.pro, L.epi)
                                         : select_bt<SIDE_COLS>(bt, L.pro, L.epi);
    if (!fn) return static_cast<int>(cudaErrorInvalidDeviceFunction);
    if (L.nvec == 0) return 0;
    const int64_t grid = (L.nvec + R - 1) / R;
    const size_t smem = static_cast<size_t>(plan.d * R +
        extra_smem_floats(R, static_cast<int>(plan.d), L.epi, L.pro, group)) * 4;
    QuantDev qd{};
    if (q) qd = *q;
    fn<<<static_cast<unsigned>(grid), NT, smem, static_cast<cudaStream_t>(stream)>>>(plan, qd, L, R);
    return static_cast<int>(cudaGetLastError());
}

int launch_quantize(const QuantDev &q, const void *in, int in_dtype, int64_t rows, int64_t cols,
                    int64_t ld_in, uint8_t *codes, uint16_t *scales, void *stream) {
    if (rows == 0) return 0;
    const int64_t items = rows * (cols / q.group);
    int64_t blocks = (items + 7) / 8;          // 8 warps per block
    if (blocks > 148 * 16) blocks = 148 * 16;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (in_dtype == HARP_F32)
        quantize_kernel<PRO_F32><<<static_cast<unsigned>(blocks), 256, 0, st>>>(q, in, rows, cols, ld_in, codes, scales);
    else
        quantize_kernel<PRO_BF16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(q, in, rows, cols, ld_in, codes, scales);
    return static_cast<int>(cudaGetLastError());
}

int launch_dequantize(const QuantDev &q, const uint8_t *codes, const uint16_t *scales,
                      int64_t rows, int64_t cols, void *out, int out_dtype, int64_t ld_out,
                      void *stream) {
    const int64_t n = rows * cols;
    if (n == 0) return 0;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (out_dtype == HARP_F32)
        dequantize_kernel<EPI_F32><<<static_cast<unsigned>(blocks), 256, 0, st>>>(q, codes, scales, rows, cols, out, ld_out);
    else
        dequantize_kernel<EPI_BF16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(q, codes, scales, rows, cols, out, ld_out);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace harp
