// harp_short.cu -- row-side calls on short vectors (d = 32, 64 or 128),
// e.g. PolarQuant's per-block rotation (gist.science paper 2603.29078,
// section 2: weight rows cut into blocks of 128, each rotated by H_128, then
// Lloyd-Max coded with the block norm as scale), and its two-stage codec
// (section 3: Q5 weights restored to FP16, then an absmax INT4 quantizer).
//
// Design: one thread owns one vector. A CTA of 256 threads takes tiles of
// 256 consecutive rows; the CTAs are persistent and while a tile is being
// computed the next tile's raw input (bf16 rows or packed codes) is already
// on its way into a shared staging buffer by cp.async, so the HBM traffic
// overlaps the arithmetic. The tile lives in shared memory as [256][d + 1]
// fp32 (odd pitch: the 32 lanes of a warp, reading the same coordinate of
// 32 different vectors, hit 32 different banks). A stage walks the thread's
// groups: it reads the b inputs of a group into registers, forms the b
// outputs in packed fp32 pairs from the block held in shared memory (every
// lane of a warp reads the same coefficients, a broadcast), and writes them
// back in place; no
// barrier is needed between stages because no thread touches another's row.
// The quantizer works per thread too; the packed codes are parked in the
// row's own (consumed) shared memory and stored with coalesced writes.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "harp_internal.h"
#include "harp_quant_dev.cuh"

namespace harp {
namespace {

using namespace dq;

constexpr int ST = 256;        // vectors per tile
constexpr int NP = 2;          // threads per vector
constexpr int NTT = ST * NP;   // threads per CTA
constexpr int SD_MAX = 128;    // longest vector handled here
constexpr int B_MAX = 32;      // largest radix handled here (registers)
constexpr int MAXCH = SD_MAX / 32 / NP;   // 32-code chunks of a row per thread
constexpr size_t SMEM_LIMIT = 232448;

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

__device__ __forceinline__ float bf16_to_f(unsigned short b) { return __uint_as_float(static_cast<unsigned>(b) << 16); }
__device__ __forceinline__ unsigned short f_to_bf16(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }

__device__ __forceinline__ float round_mid(float v, int mid) {
    if (mid == HARP_BF16) return bf16_to_f(f_to_bf16(v));
    if (mid == HARP_F16) return __half2float(__float2half_rn(fminf(fmaxf(v, -65504.0f), 65504.0f)));
    return v;
}

// Shared-memory layout (in 4-byte words), the same on host and device.
struct ShortLayout {
    int xp;          // tile row pitch (d + 1)
    int x_words;     // ST * xp
    int coef_off, coef_words;
    int coef_total;  // words of all stages' blocks (coef_words rounds it up)
    int sign_off;    // d words
    int tab_off;     // 32 levels, 32 thresholds (+inf past the last), 256 bin bytes
    int red_off;     // [NP][4][ST] partial group statistics
    int stage_off;   // staging buffer
    int stage_pitch; // words per staged row
    int total_words;
};

__host__ __device__ inline ShortLayout short_layout(const PlanDev &P, int mode, int in_bits) {
    ShortLayout L{};
    const int d = static_cast<int>(P.d);
    L.xp = d + 1;
    L.x_words = ST * L.xp;
    L.coef_off = L.x_words;
    int cw = 0;
    for (int t = 0; t < P.m; ++t) cw += static_cast<int>(d / P.st[t].b) * P.st[t].b * P.st[t].kpad;
    L.coef_total = cw;
    L.coef_words = (cw + 3) & ~3;
    L.sign_off = L.coef_off + L.coef_words;
    L.tab_off = L.sign_off + ((d + 3) & ~3);
    L.red_off = L.tab_off + 64 + 64;
    L.stage_off = L.red_off + NP * 4 * ST;
    // bf16 rows: d/2 words padded to a multiple of 4 plus 4 (16-byte rows
    // whose 16-byte reads by 8 neighbouring lanes cover all 32 banks);
    // codes: d*bits/32 words rounded up to an odd count (conflict-free
    // 4-byte reads).
    L.stage_pitch = (mode == SHORT_FWD) ? ((d / 2 + 3) & ~3) + 4 : ((d * in_bits / 32) | 1);
    L.total_words = L.stage_off + ST * L.stage_pitch;
    return L;
}

// Packed fp32 pairs: one instruction does two IEEE single-precision FMAs,
// each half rounding exactly like fmaf.
typedef unsigned long long f2_t;

__device__ __forceinline__ f2_t f2_pack(float lo, float hi) {
    f2_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(f2_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ f2_t f2_fma(f2_t a, f2_t b, f2_t c) {
    f2_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Blocks of stage t for the direction, input-major: row j (kpad floats)
// holds the coefficient of input j in every output. Forward applies B
// (plan layout fwd[c][j][k] = B[k][j]); inverse applies B^T (plan layout
// inv[c][k][j] = B[k][j]: input k, output j).
__device__ __forceinline__ const float *stage_cols(const StageDev &S, bool fwd) { return fwd ? S.fwd : S.inv; }

// One stage on one thread's row: for every group (h, l), with inputs
// x_j = row[h*b*s + j*s + l], output o = sum_j C[c][j][o] x_j (j in order,
// one rounding per FMA), written back in place. Outputs are accumulated in
// packed pairs, input by input, so consecutive FMAs are independent.
// BM >= max(b, 4) is the register width; padding coefficients are zero.
template <int BM, bool EXACT>
__device__ __forceinline__ void stage_row(float *xr, const float *C, int b_rt, int kpad, int s, int d, int part) {
    const int b = EXACT ? BM : b_rt;      // b == BM: every guard below folds away
    const int nh = d / (b * s);
    int cidx = 0;
    for (int h = 0; h < nh; ++h) {
        for (int l = 0; l < s; ++l, ++cidx) {
            if ((cidx & (NP - 1)) != part) continue;      // the row's groups alternate between its threads
            const float *cr = C + cidx * b * kpad;
            float *base = xr + h * b * s + l;
            float x[BM];
#pragma unroll
            for (int j = 0; j < BM; ++j) x[j] = (j < b) ? base[j * s] : 0.0f;
            f2_t acc[BM / 2];
#pragma unroll
            for (int p = 0; p < BM / 2; ++p) acc[p] = 0ull;      // (+0.0f, +0.0f)
#pragma unroll
            for (int j = 0; j < BM; ++j) {
                if (j < b) {
                    const f2_t xx = f2_pack(x[j], x[j]);
                    const ulonglong2 *w = reinterpret_cast<const ulonglong2 *>(cr + j * kpad);
#pragma unroll
                    for (int q = 0; q < BM / 4; ++q) {
                        if (4 * q < b) {
                            const ulonglong2 wq = w[q];
                            acc[2 * q] = f2_fma(wq.x, xx, acc[2 * q]);
                            acc[2 * q + 1] = f2_fma(wq.y, xx, acc[2 * q + 1]);
                        }
                    }
                }
            }
#pragma unroll
            for (int p = 0; p < BM / 2; ++p) {
                float lo, hi;
                f2_unpack(acc[p], lo, hi);
                if (2 * p < b) base[(2 * p) * s] = lo;
                if (2 * p + 1 < b) base[(2 * p + 1) * s] = hi;
            }
        }
    }
}

// A stage whose blocks are all the normalised Sylvester Hadamard matrix H_b
// (HARP section 2.2, theta = 0; PolarQuant section 2's H_128 is the product
// of such stages): the fast Walsh-Hadamard butterfly, log2 b rounds of
// (a + c, a - c) on inputs h apart, gives sum_j (-1)^popcount(k & j) x_j for
// every output k; one multiply by the block entry 1/sqrt(b) follows. H_b is
// symmetric, so the same code serves the inverse (B^T = B).
template <int B>
__device__ __forceinline__ void stage_row_fwht(float *xr, int s, int d, int part) {
    const float scale = static_cast<float>(1.0 / sqrt(static_cast<double>(B)));
    const int nh = d / (B * s);
    int cidx = 0;
    for (int h = 0; h < nh; ++h) {
        for (int l = 0; l < s; ++l, ++cidx) {
            if ((cidx & (NP - 1)) != part) continue;
            float *base = xr + h * B * s + l;
            float x[B];
#pragma unroll
            for (int j = 0; j < B; ++j) x[j] = base[j * s];
#pragma unroll
            for (int hh = 1; hh < B; hh <<= 1)
#pragma unroll
                for (int i = 0; i < B; ++i)
                    if ((i & hh) == 0) {
                        const float a = x[i], c = x[i + hh];
                        x[i] = a + c;
                        x[i + hh] = a - c;
                    }
#pragma unroll
            for (int j = 0; j < B; ++j) base[j * s] = x[j] * scale;
        }
    }
}

// HAD_ONLY: a build for processors whose every stage is all-Sylvester
// (PolarQuant's H_128), carrying only the butterflies, so the hot loop's code
// stays small (the general build's FMA stages of every width crowd the
// instruction cache).
template <bool HAD_ONLY>
__device__ __forceinline__ void run_stage_row(float *xr, const float *C, const StageDev &S, int d, int part) {
    const int b = S.b, kp = S.kpad, s = static_cast<int>(S.s);
    if (HAD_ONLY || S.had) {
        switch (b) {
            case 2: stage_row_fwht<2>(xr, s, d, part); return;
            case 4: stage_row_fwht<4>(xr, s, d, part); return;
            case 8: stage_row_fwht<8>(xr, s, d, part); return;
            case 16: stage_row_fwht<16>(xr, s, d, part); return;
            case 32: stage_row_fwht<32>(xr, s, d, part); return;
            default: break;
        }
    }
    if constexpr (HAD_ONLY) return;
    switch (b) {
        case 4: stage_row<4, true>(xr, C, b, kp, s, d, part); break;
        case 8: stage_row<8, true>(xr, C, b, kp, s, d, part); break;
        case 16: stage_row<16, true>(xr, C, b, kp, s, d, part); break;
        case 32: stage_row<32, true>(xr, C, b, kp, s, d, part); break;
        default:
            if (b <= 4) stage_row<4, false>(xr, C, b, kp, s, d, part);
            else if (b <= 8) stage_row<8, false>(xr, C, b, kp, s, d, part);
            else if (b <= 16) stage_row<16, false>(xr, C, b, kp, s, d, part);
            else stage_row<B_MAX, false>(xr, C, b, kp, s, d, part);
    }
}

// One of the 4 values a[0..3] picked by a runtime index (registers only).
__device__ __forceinline__ float pick4(const float (&a)[4], int i) {
    return i == 0 ? a[0] : i == 1 ? a[1] : i == 2 ? a[2] : a[3];
}

// Quantise the tile's rows; thread (v, part) owns chunks part, part + NP, ...
// of row v (32 codes each). Group statistics: each thread sums (or maxes)
// its chunks of every group in order, the NP partials meet in shared memory
// and are combined in part order. Codes are formed in registers; after a
// barrier (every value of the row has been read) the packed words of chunk k
// go to words [k*BITS, k*BITS + BITS) of the row's own shared memory.
// Called by every thread of the CTA (it holds barriers).
template <int BITS>
__device__ __forceinline__ void quantize_rows(float *xr, const QuantDev &Q, const float *thr,
                                              const unsigned char *bins, bool use_bins, int d, int part,
                                              float *red, int v, bool mine, uint16_t *scales_row) {
    const int g = Q.group, ngr = d / g, nch = d / 32, lcpg = __ffs(g / 32) - 1;
    const bool is_max = Q.stat_max != 0;            // group statistic: max |x| or sum of squares
    const bool lm = (Q.kind == HARP_LLOYD_MAX);
    float st[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ci = 0; ci < MAXCH; ++ci) {
        const int ck = part + ci * NP;
        if (mine && ck < nch) {
            const int q = ck >> lcpg;
            float a = pick4(st, q);
            for (int e = 0; e < 32; ++e) a = combine(a, xr[ck * 32 + e], is_max);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
                if (qq == q) st[qq] = a;
        }
    }
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) red[(part * 4 + qq) * ST + v] = st[qq];
    __syncthreads();
    float sc[4] = {0.f, 0.f, 0.f, 0.f}, inv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
        if (mine && qq < ngr) {
            float tot = red[qq * ST + v];
#pragma unroll
            for (int pp = 1; pp < NP; ++pp) {
                const float o = red[(pp * 4 + qq) * ST + v];
                tot = is_max ? fmaxf(tot, o) : tot + o;
            }
            const unsigned short hb = group_scale_bits(tot, Q);
            if (part == 0) scales_row[qq] = hb;
            sc[qq] = __half2float(__ushort_as_half(hb));
            inv[qq] = (sc[qq] > 0.0f) ? __frcp_rn(sc[qq]) : 0.0f;
        }
    }
    unsigned w[MAXCH][BITS];
#pragma unroll
    for (int ci = 0; ci < MAXCH; ++ci) {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[ci][i] = 0u;
        const int ck = part + ci * NP;
        if (mine && ck < nch) {
            const int q = ck >> lcpg;
            const float s = pick4(sc, q), is = pick4(inv, q);
            // one of two whole loops, so only one code path is fetched and run
            if (use_bins && s > 0.0f) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const unsigned code = static_cast<unsigned>(code_binned<256>(xr[ck * 32 + e] * is, thr, bins));
                    const int bit = e * BITS, wi = bit >> 5, sh = bit & 31;
                    w[ci][wi] |= code << sh;
                    if (sh + BITS > 32) w[ci][wi + 1] |= code >> (32 - sh);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const unsigned code = static_cast<unsigned>(
                        code_of_smem<BITS>(xr[ck * 32 + e], s, is, lm, thr));
                    const int bit = e * BITS, wi = bit >> 5, sh = bit & 31;
                    w[ci][wi] |= code << sh;
                    if (sh + BITS > 32) w[ci][wi + 1] |= code >> (32 - sh);
                }
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int ci = 0; ci < MAXCH; ++ci) {
        const int ck = part + ci * NP;
        if (mine && ck < nch) {
            unsigned *dst = reinterpret_cast<unsigned *>(xr) + ck * BITS;
#pragma unroll
            for (int i = 0; i < BITS; ++i) dst[i] = w[ci][i];
        }
    }
}

template <int BITS>
__device__ __forceinline__ void decode_row(float *xr, const unsigned *src, const float *lev, const float *sc,
                                           int g, int d, int part) {
    constexpr unsigned MASK = (1u << BITS) - 1u;
    for (int ch = part; ch < d / 32; ch += NP) {
        unsigned w[BITS];
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = src[ch * BITS + i];
        const int q = (ch * 32) / g;           // scale group of this chunk (< 4)
        const float s = q == 0 ? sc[0] : q == 1 ? sc[1] : q == 2 ? sc[2] : sc[3];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int bit = e * BITS, wi = bit >> 5, sh = bit & 31;
            unsigned code = w[wi] >> sh;
            if (sh + BITS > 32) code |= w[wi + 1] << (32 - sh);
            xr[ch * 32 + e] = s * lev[code & MASK];
        }
    }
}

// Coalesced store of the tile's packed code words: the rows v0 .. v0+nv-1
// are contiguous in global memory, row r's words parked at the start of
// shared row r.
template <int BITS>
__device__ __forceinline__ void store_codes(const float *X, int xp, int d, int64_t v0, int nv, uint8_t *codes,
                                            int tid) {
    const int wpr = d / 32 * BITS;           // words per row
    unsigned *dst = reinterpret_cast<unsigned *>(codes) + v0 * wpr;
    const int n = nv * wpr;
    const int dk = d / 32;
    for (int i = tid; i < n; i += NTT) {
        const int r = (i / BITS) / dk, k = i - r * wpr;
        dst[i] = reinterpret_cast<const unsigned *>(X)[r * xp + k];
    }
}

template <int MODE, bool HAD_ONLY>
__global__ void __launch_bounds__(NTT, 1)
short_kernel(const PlanDev P, const QuantDev Q, const ShortLaunch L) {
    extern __shared__ float4 smem_f4[];
    float *sm = reinterpret_cast<float *>(smem_f4);
    const int tid = threadIdx.x;
    const int v = tid & (ST - 1), part = tid / ST;   // the thread's vector and its share of it
    const int d = static_cast<int>(P.d);
    const int in_bits = (MODE == SHORT_FWD) ? 0 : Q.bits;
    const ShortLayout Y = short_layout(P, MODE, in_bits);
    float *X = sm;
    float *C = sm + Y.coef_off;
    float *sg = sm + Y.sign_off;
    float *lev = sm + Y.tab_off;
    float *thr = lev + 32;
    unsigned char *bins = reinterpret_cast<unsigned char *>(lev + 64);
    float *red = sm + Y.red_off;
    unsigned *stg = reinterpret_cast<unsigned *>(sm + Y.stage_off);
    const bool fwd = (MODE == SHORT_FWD);
    const QuantDev &QO = (MODE == SHORT_REQUANT) ? L.q2 : Q;   // the quantizer of the epilogue

    // per-CTA constants: blocks of every stage, signs, tables
    {
        int off = 0;
        for (int t = 0; t < P.m; ++t) {
            const StageDev &S = P.st[t];
            const int n4 = static_cast<int>(d / S.b) * S.b * S.kpad / 4;
            const float4 *src = reinterpret_cast<const float4 *>(stage_cols(S, fwd));
            for (int i = tid; i < n4; i += NTT) reinterpret_cast<float4 *>(C + off)[i] = __ldg(src + i);
            off += n4 * 4;
        }
        for (int i = tid; i < d; i += NTT) sg[i] = __ldg(P.signs + i);
        const int K = 1 << QO.bits;
        if (tid < 32) {
            lev[tid] = Q.level[tid];
            thr[tid] = (tid < K - 1) ? QO.thr[tid] : __int_as_float(0x7f800000);
        }
        if (L.bins && tid < 256) bins[tid] = bin_entry<256>(tid, QO.thr, K);
    }

    const int64_t ntiles = (L.nvec + ST - 1) / ST;
    const int ld = __ffs(d) - 1;                      // d is a power of two
    const int wpr_in = (MODE == SHORT_FWD) ? 0 : d / 32 * in_bits;
    const int ng_in = (MODE == SHORT_FWD) ? 1 : d / Q.group;
    float sc_next[4] = {0.f, 0.f, 0.f, 0.f};

    auto issue = [&](int64_t tile) {
        const int64_t v0 = tile * ST;
        const int nv = (L.nvec - v0 < ST) ? static_cast<int>(L.nvec - v0) : ST;
        if constexpr (MODE == SHORT_FWD) {
            const int gsh = ld - 3;                       // 16-byte granules per row: d / 8
            const int gpr = 1 << gsh;
            const unsigned short *src = static_cast<const unsigned short *>(L.in);
            for (int i = tid; i < nv * gpr; i += NTT) {
                const int r = i >> gsh, k = i & (gpr - 1);
                cp_async16(stg + r * Y.stage_pitch + k * 4, src + (v0 + r) * d + k * 8);
            }
        } else {
            // one warp per row, lanes over the row's words
            const unsigned *src = reinterpret_cast<const unsigned *>(L.in_codes);
            for (int r = tid >> 5; r < nv; r += NTT / 32)
                for (int k = tid & 31; k < wpr_in; k += 32)
                    cp_async4(stg + r * Y.stage_pitch + k, src + (v0 + r) * wpr_in + k);
            if (v < nv) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (q < ng_in)
                        sc_next[q] = __half2float(__ushort_as_half(__ldg(L.in_scales + (v0 + v) * ng_in + q)));
            }
        }
        cp_async_commit();
    };

    if (blockIdx.x < ntiles) issue(blockIdx.x);
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t v0 = tile * ST;
        const int nv = (L.nvec - v0 < ST) ? static_cast<int>(L.nvec - v0) : ST;
        const bool mine = v < nv;
        float *xr = X + v * Y.xp;
        cp_async_wait_all();
        __syncthreads();            // staging landed; previous tile's readers of X are done
        float sc[4] = {sc_next[0], sc_next[1], sc_next[2], sc_next[3]};
        if (mine) {
            if constexpr (MODE == SHORT_FWD) {
                const uint4 *row = reinterpret_cast<const uint4 *>(stg + v * Y.stage_pitch);
                for (int k = part; k < d / 8; k += NP) {
                    const uint4 u = row[k];
                    const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        xr[8 * k + 2 * e] = __uint_as_float(w[e] << 16) * sg[8 * k + 2 * e];
                        xr[8 * k + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u) * sg[8 * k + 2 * e + 1];
                    }
                }
            } else {
                const unsigned *row = stg + v * Y.stage_pitch;
                switch (in_bits) {
                    case 2: decode_row<2>(xr, row, lev, sc, Q.group, d, part); break;
                    case 3: decode_row<3>(xr, row, lev, sc, Q.group, d, part); break;
                    case 4: decode_row<4>(xr, row, lev, sc, Q.group, d, part); break;
                    default: decode_row<5>(xr, row, lev, sc, Q.group, d, part); break;
                }
            }
        }
        __syncthreads();            // staging consumed, rows complete
        if (tile + gridDim.x < ntiles) issue(tile + gridDim.x);

        if (fwd) {
            int o = 0;
            for (int t = 0; t < P.m; ++t) {
                if (mine) run_stage_row<HAD_ONLY>(xr, C + o, P.st[t], d, part);
                __syncthreads();
                o += static_cast<int>(d / P.st[t].b) * P.st[t].b * P.st[t].kpad;
            }
        } else {
            int o = Y.coef_total;
            for (int t = P.m - 1; t >= 0; --t) {
                o -= static_cast<int>(d / P.st[t].b) * P.st[t].b * P.st[t].kpad;
                if (mine) run_stage_row<HAD_ONLY>(xr, C + o, P.st[t], d, part);
                __syncthreads();
            }
            if (mine) {
                for (int i = part; i < d; i += NP) {
                    float x = xr[i] * sg[i];
                    if constexpr (MODE == SHORT_REQUANT) x = round_mid(x, L.mid);
                    xr[i] = x;
                }
            }
            __syncthreads();
        }

        // values out (inverse result, rotated copy or restored weights)
        void *vout = L.out;
        if (vout) {
            // one warp per row, each lane a pair of neighbouring columns:
            // 32-bit stores of two 16-bit values, 64-bit stores of two floats
            const int odt = L.out_dtype, lane = tid & 31;
            for (int r = tid >> 5; r < nv; r += NTT / 32) {
                const float *xs = X + r * Y.xp;
                const int64_t off = (v0 + r) * d;
                for (int c = 2 * lane; c < d; c += 64) {
                    const float a = xs[c], b = xs[c + 1];
                    if (odt == HARP_F32) {
                        *reinterpret_cast<float2 *>(static_cast<float *>(vout) + off + c) = make_float2(a, b);
                    } else if (odt == HARP_BF16) {
                        *reinterpret_cast<unsigned *>(static_cast<unsigned short *>(vout) + off + c) =
                            f_to_bf16(a) | (static_cast<unsigned>(f_to_bf16(b)) << 16);
                    } else {
                        *reinterpret_cast<__half2 *>(static_cast<__half *>(vout) + off + c) =
                            __halves2half2(__float2half_rn(a), __float2half_rn(b));
                    }
                }
            }
        }
        if constexpr (MODE != SHORT_INV) {
            // (quantize_rows reads X only after its first barrier; the row
            // stores above read X too and never write it)
            uint16_t *srow = L.scales + (v0 + v) * (d / QO.group);
            switch (QO.bits) {
                case 2: quantize_rows<2>(xr, QO, thr, bins, L.bins, d, part, red, v, mine, srow); break;
                case 3: quantize_rows<3>(xr, QO, thr, bins, L.bins, d, part, red, v, mine, srow); break;
                case 4: quantize_rows<4>(xr, QO, thr, bins, L.bins, d, part, red, v, mine, srow); break;
                default: quantize_rows<5>(xr, QO, thr, bins, L.bins, d, part, red, v, mine, srow); break;
            }
            __syncthreads();
            switch (QO.bits) {
                case 2: store_codes<2>(X, Y.xp, d, v0, nv, L.codes, tid); break;
                case 3: store_codes<3>(X, Y.xp, d, v0, nv, L.codes, tid); break;
                case 4: store_codes<4>(X, Y.xp, d, v0, nv, L.codes, tid); break;
                default: store_codes<5>(X, Y.xp, d, v0, nv, L.codes, tid); break;
            }
        }
    }
    cp_async_wait_all();
}

template <bool H>
const void *short_fn(int mode) {
    return (mode == SHORT_FWD) ? reinterpret_cast<const void *>(short_kernel<SHORT_FWD, H>)
         : (mode == SHORT_INV) ? reinterpret_cast<const void *>(short_kernel<SHORT_INV, H>)
                               : reinterpret_cast<const void *>(short_kernel<SHORT_REQUANT, H>);
}

template <bool H>
void short_run(int mode, unsigned grid, size_t smem, cudaStream_t st, const PlanDev &P, const QuantDev &q,
               const ShortLaunch &L) {
    if (mode == SHORT_FWD) short_kernel<SHORT_FWD, H><<<grid, NTT, smem, st>>>(P, q, L);
    else if (mode == SHORT_INV) short_kernel<SHORT_INV, H><<<grid, NTT, smem, st>>>(P, q, L);
    else short_kernel<SHORT_REQUANT, H><<<grid, NTT, smem, st>>>(P, q, L);
}

}  // namespace

size_t short_smem_bytes(const PlanDev &P, int mode, int in_bits) {
    return static_cast<size_t>(short_layout(P, mode, in_bits).total_words) * 4;
}

bool short_ok(const PlanDev &P, int mode, int in_bits) {
    if (P.d != 32 && P.d != 64 && P.d != SD_MAX) return false;
    for (int t = 0; t < P.m; ++t)
        if (P.st[t].b > B_MAX) return false;
    return short_smem_bytes(P, mode, in_bits) <= SMEM_LIMIT;
}

int launch_short(const PlanDev &P, const QuantDev &q, const ShortLaunch &Lin, void *stream) {
    if (Lin.nvec == 0) return cudaSuccess;
    ShortLaunch L = Lin;
    L.bins = (L.mode == SHORT_INV) ? 0 : (bins_exact(L.mode == SHORT_REQUANT ? L.q2 : q, 256) ? 1 : 0);
    const int in_bits = (L.mode == SHORT_FWD) ? 0 : q.bits;
    const size_t smem = short_smem_bytes(P, L.mode, in_bits);
    bool had_only = true;            // every stage all-Sylvester: the butterfly-only build
    for (int t = 0; t < P.m; ++t) had_only = had_only && P.st[t].had && P.st[t].b <= B_MAX;
    const void *fn = had_only ? short_fn<true>(L.mode) : short_fn<false>(L.mode);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, NTT, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t ntiles = (L.nvec + ST - 1) / ST;
    const int64_t grid = ntiles < static_cast<int64_t>(sms) * per_sm ? ntiles : static_cast<int64_t>(sms) * per_sm;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (had_only) short_run<true>(L.mode, static_cast<unsigned>(grid), smem, st, P, q, L);
    else short_run<false>(L.mode, static_cast<unsigned>(grid), smem, st, P, q, L);
    return cudaGetLastError();
}

}  // namespace harp
