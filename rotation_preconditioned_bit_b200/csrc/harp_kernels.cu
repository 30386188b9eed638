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
#include "harp_quant_dev.cuh"

namespace harp {
namespace {

using namespace dq;

constexpr int NT = 256;              // threads per CTA (up to 255 registers each)
constexpr int SMEM_MAX = 232448;     // opt-in dynamic shared memory per CTA (227 KB)

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

// A value rounded (nearest even) to the restored weights' storage type:
// float, bfloat16, or fp16 saturating at +-65504.
__device__ __forceinline__ float round_mid(float v, int mid) {
    if (mid == HARP_BF16) return bf16_bits_to_float(float_to_bf16_bits(v));
    if (mid == HARP_F16) return __half2float(__float2half_rn(fminf(fmaxf(v, -65504.0f), 65504.0f)));
    return v;
}

// Store a value already rounded by round_mid (the conversion is exact).
__device__ __forceinline__ void store_mid(void *base, int64_t off, float v, int mid) {
    if (mid == HARP_BF16) static_cast<unsigned short *>(base)[off] = float_to_bf16_bits(v);
    else if (mid == HARP_F16) static_cast<__half *>(base)[off] = __float2half_rn(v);
    else static_cast<float *>(base)[off] = v;
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

// ------------------------------------------------------------ tile geometry

// Shared-memory tile of R vectors: coordinate i's R floats start at
//   row(i) = i * Rp + padq * (i / bl)
// with bl the last radix of the schedule. The 4-float pad after every last-
// radix group puts neighbouring groups of the last stage (which are bl
// coordinates apart) on different banks; every stage's group then has an
// affine address a0 + j * Sj in its input index j.
struct Geo {
    int d, R, Rp, padq, bl, bl_shift;
    __device__ __forceinline__ int div_bl(int i) const { return bl_shift >= 0 ? (i >> bl_shift) : (i / bl); }
    __device__ __forceinline__ int row(int i) const { return i * Rp + padq * div_bl(i); }
};

// ------------------------------------------------------------ stage core

template <int VW>
__device__ __forceinline__ void ldsv(const float *p, float (&v)[VW]) {
    if constexpr (VW == 4) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else if constexpr (VW == 2) {
        const float2 t = *reinterpret_cast<const float2 *>(p);
        v[0] = t.x; v[1] = t.y;
    } else {
        v[0] = *p;
    }
}

template <int VW>
__device__ __forceinline__ void stsv(float *p, const float *v) {
    if constexpr (VW == 4) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (VW == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    } else {
        *p = v[0];
    }
}

// Coefficients j0 .. j0+CJ-1 of rows k0 .. k0+KL-1 of group c: for the
// forward direction rows of B (output k, inputs j), for the inverse columns
// of B. Rows past b, inputs past b and groups past the end read as zero.
constexpr int CJ = 8;   // inputs per coefficient chunk

template <int KL>
__device__ __forceinline__ void load_chunk(const float *__restrict__ rows, int c, int ngroups, int b,
                                           int kpad, int k0, int j0, bool active, float (&dst)[KL][CJ]) {
#pragma unroll
    for (int k = 0; k < KL; ++k) {
        const bool ok = active && (c < ngroups) && (k0 + k < b);
        const float4 *p = reinterpret_cast<const float4 *>(
            rows + (static_cast<size_t>(ok ? c : 0) * b + (ok ? k0 + k : 0)) * kpad + j0);
#pragma unroll
        for (int q = 0; q < CJ / 4; ++q) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (ok && j0 + q * 4 < b) v = __ldg(p + q);
            dst[k][4 * q + 0] = v.x; dst[k][4 * q + 1] = v.y;
            dst[k][4 * q + 2] = v.z; dst[k][4 * q + 3] = v.w;
        }
    }
}

// acc[k][v] += sum_{j < jn} w[k][j] * X[a + j*Sj + v] for one chunk of <= CJ
// inputs. FULL chunks carry no per-input guard: a guard inside the unrolled
// loop keeps the compiler from scheduling the shared loads ahead of the FMAs
// and halves the FMA rate.
template <int VW, int NV, int KL, bool FULL>
__device__ __forceinline__ void chunk_fma(const float *X, int a, int Sj, int jn, const float (&w)[KL][CJ],
                                          float (&acc)[KL][VW * NV]) {
#pragma unroll
    for (int j = 0; j < CJ; ++j) {
        if (FULL || j < jn) {
            const float *xp = X + a + j * Sj;
            float x[NV][VW];
#pragma unroll
            for (int n = 0; n < NV; ++n) ldsv<VW>(xp + n * VW, x[n]);
#pragma unroll
            for (int k = 0; k < KL; ++k) {
                const float wk = w[k][j];
#pragma unroll
                for (int n = 0; n < NV; ++n)
#pragma unroll
                    for (int e = 0; e < VW; ++e) acc[k][n * VW + e] = fmaf(wk, x[n][e], acc[k][n * VW + e]);
            }
        }
    }
}

// Per-stage constants of the coefficient stream of one thread.
struct StageIt {
    const float *rows;
    int b, kpad, s, s_shift, Sj, k0, qi, Gr, ngroups, nc;
    bool active;
};

// One element e of the thread's coefficient stream: chunk (e % nc) of round
// (e / nc). Prefetches element e+1 into `nxt`, accumulates this chunk from
// `cur`; after a round's last chunk: barrier, then the outputs are written
// in place over the group's inputs.
template <int VW, int NV, int KL>
__device__ __forceinline__ void stream_step(float *X, const Geo &g, const StageIt &it, int e, int total,
                                            float (&cur)[KL][CJ], float (&nxt)[KL][CJ],
                                            float (&acc)[KL][VW * NV], int &a0) {
    const int r = e / it.nc, ch = e - r * it.nc;
    if (e + 1 < total) {
        const int r1 = (ch + 1 == it.nc) ? r + 1 : r;
        const int ch1 = (ch + 1 == it.nc) ? 0 : ch + 1;
        load_chunk<KL>(it.rows, r1 * it.Gr + it.qi, it.ngroups, it.b, it.kpad, it.k0, ch1 * CJ, it.active, nxt);
    }
    const int c = r * it.Gr + it.qi;
    const bool ok = it.active && (c < it.ngroups);
    if (ch == 0) {
#pragma unroll
        for (int k = 0; k < KL; ++k)
#pragma unroll
            for (int v = 0; v < VW * NV; ++v) acc[k][v] = 0.0f;
        if (ok) {
            const int h = (it.s_shift >= 0) ? (c >> it.s_shift) : (c / it.s);
            const int l = c - h * it.s;
            a0 = g.row(h * it.b * it.s + l);
        }
    }
    if (ok) {
        const int jn = it.b - ch * CJ;
        if (jn >= CJ) chunk_fma<VW, NV, KL, true>(X, a0 + ch * CJ * it.Sj, it.Sj, CJ, cur, acc);
        else chunk_fma<VW, NV, KL, false>(X, a0 + ch * CJ * it.Sj, it.Sj, jn, cur, acc);
    }
    if (ch + 1 == it.nc) {
        __syncthreads();
        if (ok) {
#pragma unroll
            for (int k = 0; k < KL; ++k) {
                if (it.k0 + k < it.b) {
                    float *yp = X + a0 + (it.k0 + k) * it.Sj;
#pragma unroll
                    for (int n = 0; n < NV; ++n) stsv<VW>(yp + n * VW, &acc[k][n * VW]);
                }
            }
        }
    }
}

// One stride stage over the whole tile. Each thread owns KL consecutive
// outputs of one group per round (all R vectors of the tile); groups are
// handed out Gr = NT / ceil(b / KL) per round. The thread's coefficients
// arrive as a stream of CJ-input chunks, always one chunk ahead.
template <int VW, int NV, int KL>
__device__ __forceinline__ void stage_core(float *X, const Geo &g, const StageDev &S, bool last,
                                           int dir, int tid) {
    StageIt it;
    it.b = S.b;
    it.kpad = S.kpad;
    it.s = static_cast<int>(S.s);
    it.s_shift = (it.s & (it.s - 1)) == 0 ? __ffs(it.s) - 1 : -1;
    const int npairs = (it.b + KL - 1) / KL;
    it.Gr = NT / npairs;
    it.ngroups = g.d / it.b;
    it.qi = tid / npairs;
    it.k0 = (tid - it.qi * npairs) * KL;
    it.active = it.qi < it.Gr;
    it.Sj = last ? g.Rp : it.s * g.Rp + g.padq * g.div_bl(it.s);
    it.rows = (dir == HARP_FWD) ? S.inv : S.fwd;
    it.nc = (it.b + CJ - 1) / CJ;
    const int nrounds = (it.ngroups + it.Gr - 1) / it.Gr;
    const int total = nrounds * it.nc;
    float bufA[KL][CJ], bufB[KL][CJ], acc[KL][VW * NV];
    int a0 = 0;
    load_chunk<KL>(it.rows, it.qi, it.ngroups, it.b, it.kpad, it.k0, 0, it.active, bufA);
    for (int e = 0; e < total; e += 2) {
        stream_step<VW, NV, KL>(X, g, it, e, total, bufA, bufB, acc, a0);
        if (e + 1 < total) stream_step<VW, NV, KL>(X, g, it, e + 1, total, bufB, bufA, acc, a0);
    }
    __syncthreads();
}

template <int VW, int NV>
__device__ __forceinline__ void run_stage(float *X, const Geo &g, const StageDev &S, bool last, int dir, int tid) {
    // outputs per thread: enough FMAs per shared load, registers permitting
    constexpr int R = VW * NV;
    constexpr int KL = (R <= 12) ? 4 : 2;
    stage_core<VW, NV, KL>(X, g, S, last, dir, tid);
}

// Scales and codes of the tile's rows (forward, rows side).
template <int VW, int BITS, bool F32OUT>
__device__ __forceinline__ void quantize_tile(const float *X, const Geo &g, const QuantDev &Q,
                                              float *sc, float *isc, const VecLaunch &L, int64_t v0,
                                              int warp, int lane) {
    constexpr int NWARP = NT / 32;
    const int d = g.d, gsz = Q.group, ng = d / gsz, nchunk = d >> 5, cpg = gsz >> 5;
    const int nrv = g.R / VW;
    const bool is_max = Q.stat_max != 0;            // group statistic: max |x| or sum of squares
    const bool lm = (Q.kind == HARP_LLOYD_MAX);
    const bool lloyd = lm;
    // pass 1: statistics and scales, one (row group of VW rows, scale group) per warp
    for (int item = warp; item < nrv * ng; item += NWARP) {
        const int gi = item / nrv, rq = item - gi * nrv;
        float st[VW];
#pragma unroll
        for (int v = 0; v < VW; ++v) st[v] = 0.0f;
#pragma unroll 4
        for (int c = 0; c < cpg; ++c) {
            float x[VW];
            ldsv<VW>(X + g.row(gi * gsz + c * 32 + lane) + rq * VW, x);
#pragma unroll
            for (int v = 0; v < VW; ++v) st[v] = combine(st[v], x[v], is_max);
        }
#pragma unroll
        for (int v = 0; v < VW; ++v) {
            const float tot = warp_reduce(st[v], is_max);
            if (lane == v) {
                const int r = rq * VW + v;
                const unsigned short hb = group_scale_bits(tot, Q);
                const float sv = __half2float(__ushort_as_half(hb));
                sc[r * ng + gi] = sv;
                isc[r * ng + gi] = (sv > 0.0f) ? __frcp_rn(sv) : 0.0f;
                const int64_t row = v0 + r;
                if (row < L.nvec) L.scales[row * ng + gi] = hb;
            }
        }
    }
    __syncthreads();
    // pass 2: codes and packing, one (row group, 32-coordinate chunk) per warp
    float t[(1 << BITS) - 1];
#pragma unroll
    for (int k = 0; k < (1 << BITS) - 1; ++k) t[k] = Q.thr[k];
    const int64_t rowbytes = static_cast<int64_t>(d) * BITS / 8;
    for (int item = warp; item < nrv * nchunk; item += NWARP) {
        const int ch = item / nrv, rq = item - ch * nrv;
        const int i = ch * 32 + lane;
        const int gi = ch / cpg;
        float x[VW];
        ldsv<VW>(X + g.row(i) + rq * VW, x);
#pragma unroll
        for (int v = 0; v < VW; ++v) {
            const int r = rq * VW + v;
            const int64_t row = v0 + r;
            const int code = code_of<BITS>(x[v], sc[r * ng + gi], isc[r * ng + gi], lloyd, t);
            const unsigned word = pack_words<BITS>(code, lane);
            if (row < L.nvec) {
                if (lane < BITS)
                    reinterpret_cast<unsigned *>(L.codes + row * rowbytes)[ch * BITS + lane] = word;
                if constexpr (F32OUT) static_cast<float *>(L.out)[row * L.ld_out + i] = x[v];
            }
        }
    }
}

// Dequantise R rows of packed codes into the tile (inverse path). One item
// is 32 consecutive codes of one row: `BITS` aligned 32-bit words and one
// scale (groups are multiples of 32 codes); items of neighbouring rows go to
// neighbouring threads so the shared-memory writes are contiguous.
template <int BITS>
__device__ __forceinline__ void load_codes(float *X, const Geo &g, const QuantDev &Q, const VecLaunch &L,
                                           const float *lev, int64_t v0, int tid) {
    constexpr int IB = 4;
    constexpr unsigned MASK = (1u << BITS) - 1u;
    const int d = g.d, R = g.R, gsz = Q.group, ng = d / gsz;
    const int nch = d >> 5;
    const int n = R * nch;
    const int64_t rowwords = static_cast<int64_t>(d) * BITS / 32;
    for (int base = tid; base < n; base += NT * IB) {
        unsigned w[IB][BITS];
        float sc[IB];
#pragma unroll
        for (int u = 0; u < IB; ++u) {
            const int idx = base + u * NT;
            const int ch = idx / R, r = idx - ch * R;
            const int64_t row = v0 + r;
            const bool ok = idx < n && row < L.nvec;
            const unsigned *src = reinterpret_cast<const unsigned *>(L.in_codes) + (ok ? row * rowwords + ch * BITS : 0);
#pragma unroll
            for (int q = 0; q < BITS; ++q) w[u][q] = ok ? __ldg(src + q) : 0u;
            sc[u] = ok ? __half2float(__ushort_as_half(__ldg(L.in_scales + row * ng + (ch * 32) / gsz))) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < IB; ++u) {
            const int idx = base + u * NT;
            if (idx < n) {
                const int ch = idx / R, r = idx - ch * R;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int bit = e * BITS, wi = bit >> 5, sh = bit & 31;
                    unsigned code = w[u][wi] >> sh;
                    if (sh + BITS > 32) code |= w[u][wi + 1] << (32 - sh);
                    X[g.row(ch * 32 + e) + r] = sc[u] * lev[code & MASK];
                }
            }
        }
    }
}

// ------------------------------------------------------------ the kernel

template <int SIDE, int VW, int NV, int PRO, int EPI>
__global__ void __launch_bounds__(NT, 1)
vec_kernel(const PlanDev P, const QuantDev Q, const VecLaunch L, const Geo g) {
    static_assert(NT == 256, "register budget assumes 256 threads");
    extern __shared__ float4 smem_f4[];
    float *X = reinterpret_cast<float *>(smem_f4);
    constexpr int R = VW * NV;
    const int tid = threadIdx.x;
    const int d = g.d;
    const int64_t v0 = static_cast<int64_t>(blockIdx.x) * R;
    const int64_t nvec = L.nvec;
    const bool fwd = (L.dir == HARP_FWD);
    const float *__restrict__ signs = P.signs;
    const int tile_floats = g.row(d - 1) + g.Rp;      // end of the padded tile

    // ---------------------------------------------------------- prologue
    // Every load loop issues IB independent global loads per thread before it
    // writes any of them to shared memory, so a CTA waits for a few DRAM
    // round trips rather than one per element.
    if constexpr (PRO == PRO_CODES) {
        float *lev = X + tile_floats;
        if (tid < 32) lev[tid] = Q.level[tid];
        __syncthreads();
        if (Q.bits == 2) load_codes<2>(X, g, Q, L, lev, v0, tid);
        else if (Q.bits == 3) load_codes<3>(X, g, Q, L, lev, v0, tid);
        else if (Q.bits == 4) load_codes<4>(X, g, Q, L, lev, v0, tid);
        else load_codes<5>(X, g, Q, L, lev, v0, tid);
    } else if constexpr (SIDE == SIDE_ROWS) {
        if (VW == 4 && (d & 3) == 0) {
            constexpr int IB = 4;
            const int nc4 = d >> 2;
            const int n = NV * nc4;
            for (int base = tid; base < n; base += NT * IB) {
                float v[IB][4][4];
                float4 sg[IB];
#pragma unroll
                for (int u = 0; u < IB; ++u) {
                    const int idx = base + u * NT;
                    const int c4 = idx / NV, rq = idx - c4 * NV;
                    sg[u] = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        const int64_t row = v0 + rq * 4 + rr;
                        if (idx < n && row < nvec) {
                            ldg4<PRO>(L.in, row * L.ld_in + c4 * 4, v[u][rr]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 4; ++e) v[u][rr][e] = 0.0f;
                        }
                    }
                    if (fwd && idx < n) sg[u] = __ldg(reinterpret_cast<const float4 *>(signs) + c4);
                }
#pragma unroll
                for (int u = 0; u < IB; ++u) {
                    const int idx = base + u * NT;
                    if (idx < n) {
                        const int c4 = idx / NV, rq = idx - c4 * NV;
                        const float se[4] = {sg[u].x, sg[u].y, sg[u].z, sg[u].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            *reinterpret_cast<float4 *>(X + g.row(c4 * 4 + e) + rq * 4) =
                                make_float4(v[u][0][e] * se[e], v[u][1][e] * se[e], v[u][2][e] * se[e], v[u][3][e] * se[e]);
                    }
                }
            }
        } else {
            constexpr int IB = 8;
            const int n = R * d;
            for (int base = tid; base < n; base += NT * IB) {
                float v[IB];
#pragma unroll
                for (int u = 0; u < IB; ++u) {
                    const int idx = base + u * NT;
                    const int r = idx / d, i = idx - r * d;
                    const int64_t row = v0 + r;
                    v[u] = (idx < n && row < nvec) ? ldg1<PRO>(L.in, row * L.ld_in + i) : 0.0f;
                    if (fwd && idx < n) v[u] *= __ldg(signs + i);
                }
#pragma unroll
                for (int u = 0; u < IB; ++u) {
                    const int idx = base + u * NT;
                    if (idx < n) {
                        const int r = idx / d, i = idx - r * d;
                        X[g.row(i) + r] = v[u];
                    }
                }
            }
        }
    } else {  // SIDE_COLS: vectors are columns v0 .. v0+R-1, coordinates are rows
        if constexpr (VW == 4) {
            constexpr int IB = 16;
            const int n = d * NV;
            for (int base = tid; base < n; base += NT * IB) {
                float v[IB][4];
                float sg[IB];
#pragma unroll
                for (int u = 0; u < IB; ++u) {
                    const int idx = base + u * NT;
                    const int i = idx / NV, bq = idx - i * NV;
                    const int64_t col = v0 + bq * 4;
                    if (idx < n && col + 3 < nvec) {
                        ldg4<PRO>(L.in, static_cast<int64_t>(i) * L.ld_in + col, v[u]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            v[u][e] = (idx < n && col + e < nvec)
                                ? ldg1<PRO>(L.in, static_cast<int64_t>(i) * L.ld_in + col + e) : 0.0f;
                    }
                    sg[u] = (fwd && idx < n) ? __ldg(signs + i) : 1.0f;
                }
#pragma unroll
                for (int u = 0; u < IB; ++u) {
                    const int idx = base + u * NT;
                    if (idx < n) {
                        const int i = idx / NV, bq = idx - i * NV;
                        *reinterpret_cast<float4 *>(X + g.row(i) + bq * 4) =
                            make_float4(v[u][0] * sg[u], v[u][1] * sg[u], v[u][2] * sg[u], v[u][3] * sg[u]);
                    }
                }
            }
        } else {
            constexpr int IB = 8;
            const int n = d * R;
            for (int base = tid; base < n; base += NT * IB) {
                float v[IB];
#pragma unroll
                for (int u = 0; u < IB; ++u) {
                    const int idx = base + u * NT;
                    const int i = idx / R, bcol = idx - i * R;
                    const int64_t col = v0 + bcol;
                    v[u] = (idx < n && col < nvec) ? ldg1<PRO>(L.in, static_cast<int64_t>(i) * L.ld_in + col) : 0.0f;
                    if (fwd && idx < n) v[u] *= __ldg(signs + i);
                }
#pragma unroll
                for (int u = 0; u < IB; ++u) {
                    const int idx = base + u * NT;
                    if (idx < n) {
                        const int i = idx / R, bcol = idx - i * R;
                        X[g.row(i) + bcol] = v[u];
                    }
                }
            }
        }
    }
    __syncthreads();

    // ---------------------------------------------------------- stages
    for (int ti = 0; ti < P.m; ++ti) {
        const int t = fwd ? ti : P.m - 1 - ti;
        run_stage<VW, NV>(X, g, P.st[t], t == P.m - 1, L.dir, tid);
    }

    // ---------------------------------------------------------- epilogue
    if constexpr (EPI == EPI_F32 || EPI == EPI_BF16) {
        if constexpr (SIDE == SIDE_ROWS) {
            if (VW == 4 && (d & 3) == 0) {
                const int nc4 = d >> 2;
                for (int idx = tid; idx < NV * nc4; idx += NT) {
                    const int c4 = idx / NV, rq = idx - c4 * NV;
                    float v[4][4];   // [row][e]
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 w = *reinterpret_cast<const float4 *>(X + g.row(c4 * 4 + e) + rq * 4);
                        const float se = fwd ? 1.0f : __ldg(signs + c4 * 4 + e);
                        v[0][e] = w.x * se; v[1][e] = w.y * se; v[2][e] = w.z * se; v[3][e] = w.w * se;
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
                    float val = X[g.row(i) + r];
                    if (!fwd) val *= __ldg(signs + i);
                    if (row < nvec) stg1<EPI>(L.out, row * L.ld_out + i, val);
                }
            }
        } else {  // SIDE_COLS
            if constexpr (VW == 4) {
                for (int idx = tid; idx < d * NV; idx += NT) {
                    const int i = idx / NV, bq = idx - i * NV;
                    const int64_t col = v0 + bq * 4;
                    const float4 w = *reinterpret_cast<const float4 *>(X + g.row(i) + bq * 4);
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
                    float val = X[g.row(i) + bcol];
                    if (!fwd) val *= __ldg(signs + i);
                    if (col < nvec) stg1<EPI>(L.out, static_cast<int64_t>(i) * L.ld_out + col, val);
                }
            }
        }
    } else if constexpr (EPI == EPI_QUANT || EPI == EPI_QUANT_F32) {
        // rows side, forward. g % 32 == 0, g | d.
        const int ng = d / Q.group;
        float *sc = X + tile_floats;                      // [R][ng] stored scale
        float *isc = sc + R * ng;                         // [R][ng] its reciprocal
        const int warp = tid >> 5, lane = tid & 31;
        constexpr bool F32OUT = (EPI == EPI_QUANT_F32);
        if (Q.bits == 2) quantize_tile<VW, 2, F32OUT>(X, g, Q, sc, isc, L, v0, warp, lane);
        else if (Q.bits == 3) quantize_tile<VW, 3, F32OUT>(X, g, Q, sc, isc, L, v0, warp, lane);
        else if (Q.bits == 4) quantize_tile<VW, 4, F32OUT>(X, g, Q, sc, isc, L, v0, warp, lane);
        else quantize_tile<VW, 5, F32OUT>(X, g, Q, sc, isc, L, v0, warp, lane);
    } else {
        // EPI_REQUANT: rows side, inverse, codes in. The tile holds the rows
        // rotated back; apply the inverse signs, round each value to the
        // restored weights' storage type (optionally stored), then quantise
        // them with the second codebook. The level table the prologue used
        // sits where the scales go; the stages' barriers ordered its last read.
        for (int idx = tid; idx < R * d; idx += NT) {
            const int r = idx / d, i = idx - r * d;
            const int64_t row = v0 + r;
            const float v = round_mid(X[g.row(i) + r] * __ldg(signs + i), L.mid);
            X[g.row(i) + r] = v;
            if (L.out && row < nvec) store_mid(L.out, row * L.ld_out + i, v, L.mid);
        }
        __syncthreads();
        const QuantDev &Q2 = L.q2;
        const int ng = d / Q2.group;
        float *sc = X + tile_floats;
        float *isc = sc + R * ng;
        const int warp = tid >> 5, lane = tid & 31;
        if (Q2.bits == 2) quantize_tile<VW, 2, false>(X, g, Q2, sc, isc, L, v0, warp, lane);
        else if (Q2.bits == 3) quantize_tile<VW, 3, false>(X, g, Q2, sc, isc, L, v0, warp, lane);
        else if (Q2.bits == 4) quantize_tile<VW, 4, false>(X, g, Q2, sc, isc, L, v0, warp, lane);
        else quantize_tile<VW, 5, false>(X, g, Q2, sc, isc, L, v0, warp, lane);
    }
}

// ------------------------------------------------------------ standalone codec

// One warp per (row, group): statistics in the same order as the fused
// epilogue (per-lane accumulation, then the xor tree), then codes and packing.
template <int PRO, int BITS>
__device__ __forceinline__ void quantize_group(const QuantDev &Q, const void *in, int64_t off,
                                               uint8_t *codes_row, uint16_t *scale, int64_t word0,
                                               int lane, const float (&t)[(1 << BITS) - 1]) {
    const int gsz = Q.group;
    const bool is_max = Q.stat_max != 0;            // group statistic: max |x| or sum of squares
    const bool lm = (Q.kind == HARP_LLOYD_MAX);
    float st = 0.0f;
    for (int c = 0; c < (gsz >> 5); ++c) st = combine(st, ldg1<PRO>(in, off + c * 32 + lane), is_max);
    st = warp_reduce(st, is_max);
    const unsigned short hb = group_scale_bits(st, Q);
    if (lane == 0) *scale = hb;
    const float s = __half2float(__ushort_as_half(hb));
    const float is = (s > 0.0f) ? __frcp_rn(s) : 0.0f;
    for (int c = 0; c < (gsz >> 5); ++c) {
        const float x = ldg1<PRO>(in, off + c * 32 + lane);
        const int code = code_of<BITS>(x, s, is, lm, t);
        const unsigned word = pack_words<BITS>(code, lane);
        if (lane < BITS) reinterpret_cast<unsigned *>(codes_row)[word0 + c * BITS + lane] = word;
    }
}

template <int PRO, int BITS>
__global__ void __launch_bounds__(256)
quantize_kernel(const QuantDev Q, const void *in, int64_t rows, int64_t cols, int64_t ld_in,
                uint8_t *codes, uint16_t *scales) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int g = Q.group;
    const int64_t ng = cols / g;
    const int64_t rowbytes = cols * BITS / 8;
    float t[(1 << BITS) - 1];
#pragma unroll
    for (int k = 0; k < (1 << BITS) - 1; ++k) t[k] = Q.thr[k];
    for (int64_t item = warp; item < rows * ng; item += nwarps) {
        const int64_t row = item / ng, gi = item - row * ng;
        quantize_group<PRO, BITS>(Q, in, row * ld_in + gi * g, codes + row * rowbytes, scales + row * ng + gi,
                                  ((gi * g) >> 5) * BITS, lane, t);
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

struct TileChoice {
    int R, VW, NV;
};

// Tile heights the kernels are built for: 4*NV vectors (NV = 1, 2, 3, 8) and
// the narrow 1- and 2-vector tiles for very long vectors.
constexpr TileChoice kTiles[] = {{32, 4, 8}, {12, 4, 3}, {8, 4, 2}, {4, 4, 1}, {2, 2, 1}, {1, 1, 1}};

int last_radix(const PlanDev &plan) { return plan.st[plan.m - 1].b; }

Geo make_geo(const PlanDev &plan, const TileChoice &t) {
    Geo g{};
    g.d = static_cast<int>(plan.d);
    g.R = t.R;
    g.Rp = t.R;
    g.padq = t.VW;
    g.bl = last_radix(plan);
    g.bl_shift = (g.bl & (g.bl - 1)) == 0 ? __builtin_ctz(static_cast<unsigned>(g.bl)) : -1;
    return g;
}

int64_t smem_floats(const PlanDev &plan, const TileChoice &t, int epi, int pro, int group) {
    const int64_t d = plan.d;
    const int bl = last_radix(plan);
    int64_t f = d * t.R + static_cast<int64_t>(t.VW) * ((d - 1) / bl);
    if (epi == EPI_QUANT || epi == EPI_QUANT_F32 || epi == EPI_REQUANT) f += 2 * t.R * (d / group);
    if (pro == PRO_CODES) f += 32;
    return f;
}

int pick_tile(const PlanDev &plan, int epi, int pro, int group) {
    for (int i = 0; i < static_cast<int>(sizeof(kTiles) / sizeof(kTiles[0])); ++i)
        if (smem_floats(plan, kTiles[i], epi, pro, group) * 4 <= SMEM_MAX) return i;
    return -1;
}

using KernelFn = void (*)(const PlanDev, const QuantDev, const VecLaunch, const Geo);

template <int SIDE, int VW, int NV, int PRO, int EPI>
KernelFn get_kernel() {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(vec_kernel<SIDE, VW, NV, PRO, EPI>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_MAX);
    });
    return attr_err == cudaSuccess ? vec_kernel<SIDE, VW, NV, PRO, EPI> : nullptr;
}

template <int SIDE, int VW, int NV>
KernelFn select_pe(int pro, int epi) {
    if constexpr (SIDE == SIDE_ROWS) {
        if (pro == PRO_CODES) {
            if (epi == EPI_F32) return get_kernel<SIDE, VW, NV, PRO_CODES, EPI_F32>();
            if (epi == EPI_BF16) return get_kernel<SIDE, VW, NV, PRO_CODES, EPI_BF16>();
            if (epi == EPI_REQUANT) return get_kernel<SIDE, VW, NV, PRO_CODES, EPI_REQUANT>();
            return nullptr;
        }
#define HARP_ROW_CASE(P)                                                              \
    if (pro == P) {                                                                   \
        if (epi == EPI_F32) return get_kernel<SIDE, VW, NV, P, EPI_F32>();            \
        if (epi == EPI_BF16) return get_kernel<SIDE, VW, NV, P, EPI_BF16>();          \
        if (epi == EPI_QUANT) return get_kernel<SIDE, VW, NV, P, EPI_QUANT>();        \
        if (epi == EPI_QUANT_F32) return get_kernel<SIDE, VW, NV, P, EPI_QUANT_F32>(); \
    }
        HARP_ROW_CASE(PRO_F32)
        HARP_ROW_CASE(PRO_BF16)
#undef HARP_ROW_CASE
        return nullptr;
    } else {
        if (pro == PRO_F32 && epi == EPI_F32) return get_kernel<SIDE, VW, NV, PRO_F32, EPI_F32>();
        if (pro == PRO_F32 && epi == EPI_BF16) return get_kernel<SIDE, VW, NV, PRO_F32, EPI_BF16>();
        if (pro == PRO_BF16 && epi == EPI_F32) return get_kernel<SIDE, VW, NV, PRO_BF16, EPI_F32>();
        if (pro == PRO_BF16 && epi == EPI_BF16) return get_kernel<SIDE, VW, NV, PRO_BF16, EPI_BF16>();
        return nullptr;
    }
}

template <int SIDE>
KernelFn select_tile(int ti, int pro, int epi) {
    switch (ti) {
        case 0: return select_pe<SIDE, 4, 8>(pro, epi);
        case 1: return select_pe<SIDE, 4, 3>(pro, epi);
        case 2: return select_pe<SIDE, 4, 2>(pro, epi);
        case 3: return select_pe<SIDE, 4, 1>(pro, epi);
        case 4: return select_pe<SIDE, 2, 1>(pro, epi);
        default: return select_pe<SIDE, 1, 1>(pro, epi);
    }
}

}  // namespace

int vec_tile(const PlanDev &plan, int epi, int group, int pro) {
    const int ti = pick_tile(plan, epi, pro, group > 0 ? group : 32);
    return ti < 0 ? 0 : kTiles[ti].R;
}

int launch_vec(const PlanDev &plan, const QuantDev *q, const VecLaunch &L, void *stream) {
    // the group that sizes the epilogue's scale arrays
    const int group = (L.epi == EPI_REQUANT) ? L.q2.group : (q ? q->group : 32);
    const int ti = pick_tile(plan, L.epi, L.pro, group);
    if (ti < 0) return static_cast<int>(cudaErrorInvalidValue);
    KernelFn fn = (L.side == HARP_RIGHT) ? select_tile<SIDE_ROWS>(ti, L.pro, L.epi)
                                         : select_tile<SIDE_COLS>(ti, L.pro, L.epi);
    if (!fn) return static_cast<int>(cudaErrorInvalidDeviceFunction);
    if (L.nvec == 0) return 0;
    const TileChoice &t = kTiles[ti];
    const int64_t grid = (L.nvec + t.R - 1) / t.R;
    const size_t smem = static_cast<size_t>(smem_floats(plan, t, L.epi, L.pro, group)) * 4;
    QuantDev qd{};
    if (q) qd = *q;
    fn<<<static_cast<unsigned>(grid), NT, smem, static_cast<cudaStream_t>(stream)>>>(plan, qd, L, make_geo(plan, t));
    return static_cast<int>(cudaGetLastError());
}

int launch_quantize(const QuantDev &q, const void *in, int in_dtype, int64_t rows, int64_t cols,
                    int64_t ld_in, uint8_t *codes, uint16_t *scales, void *stream) {
    if (rows == 0) return 0;
    const int64_t items = rows * (cols / q.group);
    int64_t blocks = (items + 7) / 8;          // 8 warps per block
    if (blocks > 148 * 16) blocks = 148 * 16;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned nb = static_cast<unsigned>(blocks);
#define HARP_QLAUNCH(P, B) quantize_kernel<P, B><<<nb, 256, 0, st>>>(q, in, rows, cols, ld_in, codes, scales)
    if (in_dtype == HARP_F32) {
        if (q.bits == 2) HARP_QLAUNCH(PRO_F32, 2);
        else if (q.bits == 3) HARP_QLAUNCH(PRO_F32, 3);
        else if (q.bits == 4) HARP_QLAUNCH(PRO_F32, 4);
        else HARP_QLAUNCH(PRO_F32, 5);
    } else {
        if (q.bits == 2) HARP_QLAUNCH(PRO_BF16, 2);
        else if (q.bits == 3) HARP_QLAUNCH(PRO_BF16, 3);
        else if (q.bits == 4) HARP_QLAUNCH(PRO_BF16, 4);
        else HARP_QLAUNCH(PRO_BF16, 5);
    }
#undef HARP_QLAUNCH
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
