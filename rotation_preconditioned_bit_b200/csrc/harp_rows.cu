// harp_rows.cu -- the row kernel of libharp (sm_100a): right-only rotate +
// quantize of whole rows (HARP's online activation rotation) fused with the
// group quantizer, for processors whose radices are 2, 4, 8 or 16 and rows of
// up to 8192 coordinates.
//
// What it computes:
//  * HARP (gist.science paper 2605.29843) section 2.1: every row r of X is
//    mapped to M r, M = B_{m-1} ... B_0 D_s; stage t applies one b_t x b_t
//    block to every group {h b s + k s + l : k < b} of coordinates (s the
//    product of the later radices); section 3: the activation side is
//    rotated online, one row (token) at a time.
//  * PolarQuant (gist.science paper 2603.29078) sections 1 and 2: group
//    scale (RMS or max|x| / divisor), fp16 scale, Lloyd-Max midpoint count or
//    rounded absmax code, packed LSB-first.
//
// Design (B200). A persistent CTA of 512 threads walks tiles of R whole rows
// held in shared memory as fp32 (sign vector applied as they arrive). The
// next tile's rows arrive by one bulk copy (cp.async.bulk, completing on an
// mbarrier) into a staging buffer while the current tile is computed. In a
// stage each thread owns one group for RT of the tile's rows (all R rows
// when there are 512 groups or more; row sets otherwise): per input j it
// reads the group's coefficient column (the b outputs' coefficients of input
// j, contiguous in the plan's layout, from L1/L2) once and applies it to
// every one of its rows with packed fp32 pairs of FMAs (two rows per
// instruction), then writes its outputs back in place. A stage's groups are
// disjoint, so no barrier is needed inside a stage. The quantizer splits each
// row's groups into chunks of 32 x CW coordinates: every warp takes chunks,
// their statistics meet in shared memory, then every chunk is coded and
// packed by the warp that owns it (32 codes -> BITS words per step).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "harp_internal.h"
#include "harp_quant_dev.cuh"
#include "harp_tc.cuh"

namespace harp {
namespace {

using namespace dq;

constexpr int RT_THREADS = 512;
constexpr int RT_WARPS = RT_THREADS / 32;
constexpr int ROWS_SMEM_BUDGET = 224 * 1024;
constexpr long long ROWS_WAIT_LIMIT = 1ll << 30;   // SM cycles (about half a second)

// Device record of bounded waits that ran out (bit 2: a row tile's input
// never arrived); read with harp_fault_status.
__device__ unsigned int g_rows_fault;

struct RowsDesc {
    int d, m, R, pitch;           // coordinates, stages, rows per tile, tile pitch (floats)
    int b[HARP_MAX_STAGES];
    int s[HARP_MAX_STAGES];
    int sl[HARP_MAX_STAGES];      // log2 s (radices are powers of two)
    int kpad[HARP_MAX_STAGES];
    int had[HARP_MAX_STAGES];     // every block is the normalised Sylvester H_b
    const float *gfwd[HARP_MAX_STAGES];  // [((j kpad/4 + k/4) G + c) 4 + k%4] = B[k][j]
    const float *signs;
    int64_t rows;
    const void *in;
    int in_bf16;
    float *out_f32;               // optional rotated copy
    uint8_t *codes;
    uint16_t *scales;
    int chunk;                    // coordinates per quantiser chunk (32 x CW)
    int fuse0;                    // stage 0 reads the staged input itself (register-block radix, not Sylvester)
    int stage_base, part_base, bar_base, lev_base;   // float offsets in shared memory
};

// The tile stores coordinate a of a row at a XOR-swizzled word of the same
// 32-word block: a ^ ((a/32) % 8 + 8 * ((a/64) % 4)). A warp then reads 32
// consecutive coordinates, 32 coordinates 8 apart, or 4 runs of 8 that are
// 64 apart (the groups of the stages of a radix-8 processor, and the
// quantizer's lanes) from 32 different banks.
__host__ __device__ __forceinline__ int sk(int a) { return a ^ (((a >> 5) & 7) | (((a >> 6) & 3) << 3)); }

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

// One stage on the tile (rows [0, nrows)) for radix 16: thread t owns group
// g = t mod GT (GT = min(groups, threads)) for rows rs, rs + RS, ... (RS =
// threads / GT row sets), RT rows at a time, and loops over groups g,
// g + threads, ... when there are more groups than threads. acc holds RT
// rows x B outputs as packed row pairs.
template <int B, int RT>
__device__ __forceinline__ void stage_rows(float *T, const RowsDesc &D, int t, int nrows, int tid) {
    const int s = D.s[t], sl = D.sl[t], kp = D.kpad[t];
    const int G = D.d / B;
    const int GT = G < RT_THREADS ? G : RT_THREADS;
    const int RS = RT_THREADS / GT;
    const int rs = tid / GT;
    if (rs >= RS) return;
    const float *coef = D.gfwd[t];
    const int pitch = D.pitch;
    for (int g = tid - rs * GT; g < G; g += GT) {
        const int h = g >> sl, l = g & (s - 1);
        const int base = h * B * s + l;
        const float4 *cp = reinterpret_cast<const float4 *>(coef) + g;   // group-interleaved blocks
        // the thread's rows rs, rs + RS, ... in blocks of RT
        for (int rb = rs; rb < nrows; rb += RT * RS) {
            f2_t acc[RT / 2][B];
#pragma unroll
            for (int p = 0; p < RT / 2; ++p)
#pragma unroll
                for (int k = 0; k < B; ++k) acc[p][k] = 0ull;
#pragma unroll 4
            for (int j = 0; j < B; ++j) {
                float c[B];
#pragma unroll
                for (int q = 0; q < B / 4; ++q) {
                    const float4 v = __ldg(cp + static_cast<int64_t>(j * (kp >> 2) + q) * G);
                    c[4 * q] = v.x;
                    c[4 * q + 1] = v.y;
                    c[4 * q + 2] = v.z;
                    c[4 * q + 3] = v.w;
                }
                const int xa = sk(base + j * s);
#pragma unroll
                for (int p = 0; p < RT / 2; ++p) {
                    const int r0 = rb + 2 * p * RS, r1 = r0 + RS;
                    const float x0 = r0 < nrows ? T[r0 * pitch + xa] : 0.0f;
                    const float x1 = r1 < nrows ? T[r1 * pitch + xa] : 0.0f;
                    const f2_t x = f2_pack(x0, x1);
#pragma unroll
                    for (int k = 0; k < B; ++k) acc[p][k] = f2_fma(f2_pack(c[k], c[k]), x, acc[p][k]);
                }
            }
#pragma unroll
            for (int p = 0; p < RT / 2; ++p) {
                const int r0 = rb + 2 * p * RS, r1 = r0 + RS;
#pragma unroll
                for (int k = 0; k < B; ++k) {
                    float y0, y1;
                    f2_unpack(acc[p][k], y0, y1);
                    const int ya = sk(base + k * s);
                    if (r0 < nrows) T[r0 * pitch + ya] = y0;
                    if (r1 < nrows) T[r1 * pitch + ya] = y1;
                }
            }
        }
    }
}

// The same stage for radices up to 8 with the group's whole block held in
// registers: cc[j][q] = (B[2q][j], B[2q+1][j]) is loaded once (all loads in
// flight together), then the thread's rows stream through it one at a time:
// y[2q..2q+1] += cc[j][q] * (x_j, x_j), packed fp32 pairs over output pairs.
template <int B, int RT>
__device__ __forceinline__ void stage_rows_rc(float *T, const RowsDesc &D, int t, int nrows, int tid) {
    static_assert(B == 2 || B == 4 || B == 8, "register-resident blocks take radices 2, 4 and 8");
    const int s = D.s[t], sl = D.sl[t], kq = D.kpad[t] >> 2;
    const int G = D.d / B;
    const int GT = G < RT_THREADS ? G : RT_THREADS;
    const int RS = RT_THREADS / GT;
    const int rs = tid / GT;
    if (rs >= RS) return;
    const int pitch = D.pitch;
    for (int g = tid - rs * GT; g < G; g += GT) {
        const int h = g >> sl, l = g & (s - 1);
        const int base = h * B * s + l;
        // group g's float4 for (input j, outputs 4q..4q+3) sits at
        // ((j * kpad/4 + q) * G + g): consecutive threads, consecutive float4s
        const float4 *cp = reinterpret_cast<const float4 *>(D.gfwd[t]) + g;
        f2_t cc[B][B / 2];
#pragma unroll
        for (int j = 0; j < B; ++j) {
#pragma unroll
            for (int q = 0; q < (B + 3) / 4; ++q) {
                const float4 v = __ldg(cp + static_cast<int64_t>(j * kq + q) * G);
                cc[j][2 * q] = f2_pack(v.x, v.y);
                if constexpr (B >= 4) cc[j][2 * q + 1] = f2_pack(v.z, v.w);
            }
        }
        int xa[B];
#pragma unroll
        for (int j = 0; j < B; ++j) xa[j] = sk(base + j * s);
#pragma unroll 2
        for (int i = 0; i < RT; ++i) {
            const int r = rs + i * RS;
            if (r >= nrows) break;
            float *row = T + r * pitch;
            float x[B];
#pragma unroll
            for (int j = 0; j < B; ++j) x[j] = row[xa[j]];
            f2_t acc[B / 2];
#pragma unroll
            for (int q = 0; q < B / 2; ++q) acc[q] = 0ull;
#pragma unroll
            for (int j = 0; j < B; ++j) {
                const f2_t xd = f2_pack(x[j], x[j]);
#pragma unroll
                for (int q = 0; q < B / 2; ++q) acc[q] = f2_fma(cc[j][q], xd, acc[q]);
            }
#pragma unroll
            for (int q = 0; q < B / 2; ++q) {
                float y0, y1;
                f2_unpack(acc[q], y0, y1);
                row[xa[2 * q]] = y0;
                row[xa[2 * q + 1]] = y1;
            }
        }
    }
}

// Stage 0 of a register-block processor straight from the staged input
// rows (bf16 or fp32, row-major, d per row): x_j = input * sign (the signs of
// the thread's group held in registers), outputs into the fp32 tile; the
// separate convert step is skipped. Same thread <-> (group, rows) map and
// arithmetic as stage_rows_rc.
template <int B, int RT>
__device__ __forceinline__ void stage0_from_input(const void *S, float *T, const RowsDesc &D, int nrows, int tid) {
    static_assert(B == 2 || B == 4 || B == 8, "register-resident blocks take radices 2, 4 and 8");
    const int s = D.s[0], sl = D.sl[0], kq = D.kpad[0] >> 2, d = D.d;
    const int G = d / B;
    const int GT = G < RT_THREADS ? G : RT_THREADS;
    const int RS = RT_THREADS / GT;
    const int rs = tid / GT;
    if (rs >= RS) return;
    const int pitch = D.pitch;
    for (int g = tid - rs * GT; g < G; g += GT) {
        const int h = g >> sl, l = g & (s - 1);
        const int base = h * B * s + l;
        const float4 *cp = reinterpret_cast<const float4 *>(D.gfwd[0]) + g;
        f2_t cc[B][B / 2];
#pragma unroll
        for (int j = 0; j < B; ++j) {
#pragma unroll
            for (int q = 0; q < (B + 3) / 4; ++q) {
                const float4 v = __ldg(cp + static_cast<int64_t>(j * kq + q) * G);
                cc[j][2 * q] = f2_pack(v.x, v.y);
                if constexpr (B >= 4) cc[j][2 * q + 1] = f2_pack(v.z, v.w);
            }
        }
        int xa[B];
        float sg[B];
#pragma unroll
        for (int j = 0; j < B; ++j) {
            xa[j] = sk(base + j * s);
            sg[j] = __ldg(D.signs + base + j * s);
        }
#pragma unroll 2
        for (int i = 0; i < RT; ++i) {
            const int r = rs + i * RS;
            if (r >= nrows) break;
            float x[B];
            if (D.in_bf16) {
                const unsigned short *src = static_cast<const unsigned short *>(S) + r * d + base;
#pragma unroll
                for (int j = 0; j < B; ++j) x[j] = __uint_as_float(static_cast<unsigned>(src[j * s]) << 16) * sg[j];
            } else {
                const float *src = static_cast<const float *>(S) + r * d + base;
#pragma unroll
                for (int j = 0; j < B; ++j) x[j] = src[j * s] * sg[j];
            }
            f2_t acc[B / 2];
#pragma unroll
            for (int q = 0; q < B / 2; ++q) acc[q] = 0ull;
#pragma unroll
            for (int j = 0; j < B; ++j) {
                const f2_t xd = f2_pack(x[j], x[j]);
#pragma unroll
                for (int q = 0; q < B / 2; ++q) acc[q] = f2_fma(cc[j][q], xd, acc[q]);
            }
            float *row = T + r * pitch;
#pragma unroll
            for (int q = 0; q < B / 2; ++q) {
                float y0, y1;
                f2_unpack(acc[q], y0, y1);
                row[xa[2 * q]] = y0;
                row[xa[2 * q + 1]] = y1;
            }
        }
    }
}

template <int B>
__device__ __forceinline__ void stage0_from_input_any(const void *S, float *T, const RowsDesc &D, int nrows, int tid) {
    const int G = D.d / B;
    const int GT = G < RT_THREADS ? G : RT_THREADS;
    const int rt = (D.R + RT_THREADS / GT - 1) / (RT_THREADS / GT);
    if (rt <= 2) stage0_from_input<B, 2>(S, T, D, nrows, tid);
    else if (rt <= 4) stage0_from_input<B, 4>(S, T, D, nrows, tid);
    else stage0_from_input<B, 8>(S, T, D, nrows, tid);
}

// A stage whose blocks are all the normalised Sylvester Hadamard matrix H_b
// (HARP section 2.2, theta = 0): per row, the fast Walsh-Hadamard butterfly
// (log2 b rounds of (a + c, a - c) on inputs h apart) and one multiply by
// 1/sqrt(b). Same thread <-> (group, rows) map as the block stages.
template <int B>
__device__ __forceinline__ void stage_rows_fwht(float *T, const RowsDesc &D, int t, int nrows, int tid) {
    const float scale = static_cast<float>(1.0 / sqrt(static_cast<double>(B)));
    const int s = D.s[t], sl = D.sl[t];
    const int G = D.d / B;
    const int GT = G < RT_THREADS ? G : RT_THREADS;
    const int RS = RT_THREADS / GT;
    const int rs = tid / GT;
    if (rs >= RS) return;
    for (int g = tid - rs * GT; g < G; g += GT) {
        const int h = g >> sl, l = g & (s - 1);
        const int base = h * B * s + l;
        for (int r = rs; r < nrows; r += RS) {
            float *row = T + r * D.pitch;
            float x[B];
#pragma unroll
            for (int j = 0; j < B; ++j) x[j] = row[sk(base + j * s)];
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
            for (int j = 0; j < B; ++j) row[sk(base + j * s)] = x[j] * scale;
        }
    }
}

// Rows per thread for a stage of radix b on R rows with G = d/b groups.
__host__ __device__ __forceinline__ int rows_per_thread(int R, int d, int b) {
    const int G = d / b;
    const int GT = G < RT_THREADS ? G : RT_THREADS;
    const int RS = RT_THREADS / GT;
    return (R + RS - 1) / RS;
}

template <int B>
__device__ __forceinline__ void stage_rows_any(float *T, const RowsDesc &D, int t, int nrows, int tid) {
    const int rt = rows_per_thread(D.R, D.d, B);
    if constexpr (B <= 8) {
        if (rt <= 2) stage_rows_rc<B, 2>(T, D, t, nrows, tid);
        else if (rt <= 4) stage_rows_rc<B, 4>(T, D, t, nrows, tid);
        else stage_rows_rc<B, 8>(T, D, t, nrows, tid);
    } else {
        stage_rows<B, 2>(T, D, t, nrows, tid);
    }
}

// Staged input rows -> fp32 tile, times the sign vector: each thread takes
// columns c..c+3 (c a multiple of 4) of every row, its signs loaded once.
__device__ __forceinline__ void convert_rows(const RowsDesc &D, const void *S, float *T, int nrows, int tid) {
    const int d = D.d;
    for (int c = 4 * tid; c < d; c += 4 * RT_THREADS) {
        const float4 sg = __ldg(reinterpret_cast<const float4 *>(D.signs + c));
        const int p0 = sk(c), p1 = sk(c + 1), p2 = sk(c + 2), p3 = sk(c + 3);
#pragma unroll 4
        for (int r = 0; r < nrows; ++r) {
            float4 x;
            if (D.in_bf16) {
                const uint2 u = *reinterpret_cast<const uint2 *>(static_cast<const unsigned short *>(S) + r * d + c);
                x = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                                __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
            } else {
                x = *reinterpret_cast<const float4 *>(static_cast<const float *>(S) + r * d + c);
            }
            float *t = T + r * D.pitch;
            t[p0] = x.x * sg.x;
            t[p1] = x.y * sg.y;
            t[p2] = x.z * sg.z;
            t[p3] = x.w * sg.w;
        }
    }
}

// Absmax code of z = x / scale: clamp to [-qmax, qmax], then the nearest
// integer with ties to even (adding 1.5 * 2^23 leaves it in the low mantissa
// bits; exact for |z| < 2^22, and the clamp keeps |z| <= qmax), plus 2^(b-1).
// The same code as rint(z) clamped; a zero scale gives inv = 0, z = 0 and
// the mid code.
template <int BITS>
__device__ __forceinline__ int absmax_code(float x, float inv) {
    constexpr int HALF = 1 << (BITS - 1);
    constexpr float QMAX = static_cast<float>(HALF - 1);
    const float z = fminf(fmaxf(x * inv, -QMAX), QMAX);
    return (__float_as_int(z + 12582912.0f) - 0x4B400000) + HALF;
}

// Quantise the tile's rows: chunks of D.chunk coordinates (whole chunks per
// group); pass 1 writes every chunk's statistic to part[], pass 2 combines a
// group's chunks (in order, one value each), scales, codes and packs. For 2
// and 4 bits a lane codes 32 / BITS consecutive coordinates into a word of
// its own (16 codes at 2 bits, 8 at 4); 3 and 5 bits pack 32 codes across
// the warp (every lane takes part: chunks are whole multiples of 32).
template <int BITS>
__device__ __forceinline__ void quantize_rows(const float *T, const RowsDesc &D, const QuantDev &Q, float *part,
                                              const float *ts, const unsigned char *bins, int bins_ok,
                                              int64_t row0, int nrows, int warp, int lane) {
    const int d = D.d, ch = D.chunk, nch = d / ch, cpg = Q.group / ch, cw = ch >> 5;
    const bool is_max = Q.stat_max != 0, lm = (Q.kind == HARP_LLOYD_MAX);
    const int items = nrows * nch;
    for (int it = warp; it < items; it += RT_WARPS) {
        const int r = it / nch, c = it - r * nch;
        const float *x = T + r * D.pitch;
        // a chunk is whole 32-word swizzle blocks, so its words hold exactly
        // its values (in another order): the statistic reads them linearly,
        // four per 16-byte load, combined in a fixed order
        const float4 *xv = reinterpret_cast<const float4 *>(x + c * ch);
        float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
        for (int e = lane; e < ch / 4; e += 32) {
            const float4 v = xv[e];
            a0 = combine(a0, v.x, is_max);
            a1 = combine(a1, v.y, is_max);
            a2 = combine(a2, v.z, is_max);
            a3 = combine(a3, v.w, is_max);
        }
        float st = is_max ? fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) : (a0 + a1) + (a2 + a3);
        st = warp_reduce(st, is_max);
        if (lane == 0) part[it] = st;
    }
    __syncthreads();
    const int64_t wpr = static_cast<int64_t>(d) * BITS / 32;
    const int ng = d / Q.group;
    uint32_t *cwords = reinterpret_cast<uint32_t *>(D.codes);
    for (int it = warp; it < items; it += RT_WARPS) {
        const int r = it / nch, c = it - r * nch;
        const int gi = c / cpg, c0 = gi * cpg;
        float st = part[r * nch + c0];
        for (int q = 1; q < cpg; ++q) {
            const float v = part[r * nch + c0 + q];
            st = is_max ? fmaxf(st, v) : st + v;
        }
        const unsigned short hb = group_scale_bits(st, Q);
        const float sc = __half2float(__ushort_as_half(hb));
        const float inv = (sc > 0.0f) ? __frcp_rn(sc) : 0.0f;
        const int64_t row = row0 + r;
        if (lane == 0 && c == c0) D.scales[row * ng + gi] = hb;
        const float *x = T + r * D.pitch;
        uint32_t *wrow = cwords + row * wpr;
        float *frow = D.out_f32 ? D.out_f32 + row * d : nullptr;
        const bool binned = lm && bins_ok && sc > 0.0f;
        if constexpr (BITS == 2 || BITS == 4) {
            // PER consecutive codes fill one 32-bit word; no cross-lane step,
            // so lanes past the chunk's end simply skip the loop
            constexpr int PER = 32 / BITS;
#pragma unroll 4
            for (int col = c * ch + PER * lane; col < (c + 1) * ch; col += 32 * PER) {
                // col .. col + PER - 1 share one 32-word block and so one
                // swizzle mask m: coordinate col + i sits at (col ^ m) ^ i
                const int blk = col >> 5;
                const int sw = col ^ ((blk & 7) | (((blk >> 1) & 3) << 3));
                float v[PER];
#pragma unroll
                for (int i = 0; i < PER; ++i) v[i] = x[sw ^ i];
                unsigned word = 0;
                if (!lm) {
#pragma unroll
                    for (int i = 0; i < PER; ++i) word |= static_cast<unsigned>(absmax_code<BITS>(v[i], inv)) << (BITS * i);
                } else if (binned) {
#pragma unroll
                    for (int i = 0; i < PER; ++i)
                        word |= static_cast<unsigned>(code_binned<64>(v[i] * inv, ts, bins)) << (BITS * i);
                } else {
#pragma unroll
                    for (int i = 0; i < PER; ++i)
                        word |= static_cast<unsigned>(code_of_smem<BITS>(v[i], sc, inv, true, ts)) << (BITS * i);
                }
                wrow[col / PER] = word;
                if (frow) {
                    float4 *f = reinterpret_cast<float4 *>(frow + col);
#pragma unroll
                    for (int i = 0; i < PER / 4; ++i) f[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
            }
        } else {
            for (int e = 0; e < cw; ++e) {
                const int col = c * ch + 32 * e + lane;
                const float v = x[sk(col)];
                const int code = !lm ? absmax_code<BITS>(v, inv)
                                 : binned ? code_binned<64>(v * inv, ts, bins) : code_of_smem<BITS>(v, sc, inv, true, ts);
                const unsigned word = pack_words<BITS>(code, lane);
                if (lane < BITS) wrow[static_cast<int64_t>(c) * cw * BITS + e * BITS + lane] = word;
                if (frow) frow[col] = v;
            }
        }
    }
}

__global__ void __launch_bounds__(RT_THREADS, 1) rows_kernel(const __grid_constant__ RowsDesc D,
                                                             const __grid_constant__ QuantDev Q, int bins_ok) {
    extern __shared__ float4 sm4[];
    float *sm = reinterpret_cast<float *>(sm4);
    float *T = sm;
    void *S = sm + D.stage_base;
    float *part = sm + D.part_base;
    float *lev = sm + D.lev_base;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + D.bar_base);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (D.rows + D.R - 1) / D.R;
    int64_t t = blockIdx.x;
    if (t >= ntiles) return;
    const int esize = D.in_bf16 ? 2 : 4;
    {
        const int K = 1 << Q.bits;
        if (tid < 32) lev[16 + tid] = (tid < K - 1) ? Q.thr[tid] : __int_as_float(0x7f800000);
        if (bins_ok && tid < 64) reinterpret_cast<unsigned char *>(lev)[tid] = bin_entry<64>(tid, Q.thr, K);
    }
    if (tid == 0) tc::mbar_init(bar, 1);
    __syncthreads();
    auto issue = [&](int64_t tile) {
        const int64_t r0 = tile * D.R;
        const int n = static_cast<int>(min(static_cast<int64_t>(D.R), D.rows - r0));
        const uint32_t bytes = static_cast<uint32_t>(n) * D.d * esize;
        tc::mbar_arrive_expect_tx(bar, bytes);
        tc::bulk_g2s(S, static_cast<const char *>(D.in) + r0 * D.d * esize, bytes, bar);
    };
    if (tid == 0) issue(t);
    uint32_t phase = 0;
    bool fault = false;
    for (; t < ntiles; t += gridDim.x) {
        const int64_t r0 = t * D.R;
        const int nrows = static_cast<int>(min(static_cast<int64_t>(D.R), D.rows - r0));
        if (!tc::mbar_wait_bounded(bar, phase, ROWS_WAIT_LIMIT)) fault = true;
        phase ^= 1u;
        if (__syncthreads_or(fault ? 1 : 0)) {
            if (tid == 0) atomicOr(&g_rows_fault, 4u);
            break;
        }
        if (D.fuse0) {
            switch (D.b[0]) {
                case 2: stage0_from_input_any<2>(S, T, D, nrows, tid); break;
                case 4: stage0_from_input_any<4>(S, T, D, nrows, tid); break;
                default: stage0_from_input_any<8>(S, T, D, nrows, tid); break;
            }
        } else {
            convert_rows(D, S, T, nrows, tid);
        }
        // the staging buffer's reads are ordered before the next bulk copy into it
        tc::fence_proxy_async();
        __syncthreads();
        if (tid == 0 && t + gridDim.x < ntiles) issue(t + gridDim.x);
        for (int st = D.fuse0 ? 1 : 0; st < D.m; ++st) {
            if (D.had[st]) {
                switch (D.b[st]) {
                    case 2: stage_rows_fwht<2>(T, D, st, nrows, tid); break;
                    case 4: stage_rows_fwht<4>(T, D, st, nrows, tid); break;
                    case 8: stage_rows_fwht<8>(T, D, st, nrows, tid); break;
                    default: stage_rows_fwht<16>(T, D, st, nrows, tid); break;
                }
                __syncthreads();
                continue;
            }
            switch (D.b[st]) {
                case 2: stage_rows_any<2>(T, D, st, nrows, tid); break;
                case 4: stage_rows_any<4>(T, D, st, nrows, tid); break;
                case 8: stage_rows_any<8>(T, D, st, nrows, tid); break;
                default: stage_rows_any<16>(T, D, st, nrows, tid); break;
            }
            __syncthreads();
        }
        const unsigned char *bins = reinterpret_cast<const unsigned char *>(lev);
        switch (Q.bits) {
            case 2: quantize_rows<2>(T, D, Q, part, lev + 16, bins, bins_ok, r0, nrows, warp, lane); break;
            case 3: quantize_rows<3>(T, D, Q, part, lev + 16, bins, bins_ok, r0, nrows, warp, lane); break;
            case 4: quantize_rows<4>(T, D, Q, part, lev + 16, bins, bins_ok, r0, nrows, warp, lane); break;
            default: quantize_rows<5>(T, D, Q, part, lev + 16, bins, bins_ok, r0, nrows, warp, lane); break;
        }
        __syncthreads();
    }
    // a tile's copy that timed out may still land: give it one more bounded
    // wait before the CTA's shared memory is released
    if (fault && tid == 0) tc::mbar_wait_bounded(bar, phase ^ 1u, ROWS_WAIT_LIMIT);
}

struct RowsGeom {
    int R, pitch, chunk, stage_base, part_base, lev_base, bar_base, smem;
};

// Tile rows and shared-memory layout for d coordinates, or R = 0 when the
// rows do not fit. R is a power of two, at most rmax (<= 8) and 64 /
// (largest radix) so a thread's accumulators fit its registers; R <= 8 also
// keeps every row of a tile inside the block stages' loops (at most 8 rows
// per thread).
RowsGeom rows_geom(const PlanDev &P, int in_dtype, const QuantDev &q, int rmax = 8) {
    RowsGeom g{};
    const int d = static_cast<int>(P.d);
    int bmax = 1;
    for (int t = 0; t < P.m; ++t) bmax = std::max(bmax, P.st[t].b);
    const int esize = in_dtype == HARP_BF16 ? 2 : 4;
    g.pitch = d + 4;
    g.chunk = std::min(q.group, 1024);
    while (q.group % g.chunk) g.chunk >>= 1;
    for (int R = std::min(rmax, 64 / bmax); R >= 1; R >>= 1) {
        g.R = R;
        g.stage_base = ((R * g.pitch) + 31) & ~31;
        g.part_base = g.stage_base + ((R * d * esize / 4 + 31) & ~31);
        g.lev_base = g.part_base + ((R * (d / g.chunk) + 3) & ~3);
        g.bar_base = g.lev_base + 48;
        g.smem = (g.bar_base + 4) * 4;
        if (g.smem <= ROWS_SMEM_BUDGET) return g;
    }
    g.R = 0;
    return g;
}

}  // namespace

bool rows_ok(const PlanDev &P, const QuantDev &q, int in_dtype, const void *in) {
    if (P.d < 64 || P.d > 8192 || P.d % 32) return false;
    if (in_dtype != HARP_BF16 && in_dtype != HARP_F32) return false;
    if (reinterpret_cast<uintptr_t>(in) % 16) return false;
    if (q.group % 32 || P.d % q.group) return false;
    for (int t = 0; t < P.m; ++t) {
        const int b = P.st[t].b;
        if (b != 2 && b != 4 && b != 8 && b != 16) return false;
    }
    return rows_geom(P, in_dtype, q).R > 0;
}

int launch_rows(const PlanDev &P, const QuantDev &q, const void *in, int in_dtype, int64_t rows, uint8_t *codes,
                uint16_t *scales, float *rotated_out, void *stream) {
    static int attr_done[64] = {};
    static int nsm[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        e = cudaFuncSetAttribute(rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ROWS_SMEM_BUDGET);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&nsm[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    if (rows == 0) return cudaSuccess;
    // tiles as small as keep every SM busy: a tile's rows go through the
    // stages one after another, so a few rows finish sooner on more SMs
    int rmax = 1;
    while (rmax < 8 && static_cast<int64_t>(rmax) * nsm[dev] < rows) rmax <<= 1;
    const RowsGeom g = rows_geom(P, in_dtype, q, rmax);
    if (g.R == 0) return cudaErrorInvalidValue;
    RowsDesc D{};
    D.d = static_cast<int>(P.d);
    D.m = P.m;
    D.R = g.R;
    D.pitch = g.pitch;
    for (int t = 0; t < P.m; ++t) {
        D.b[t] = P.st[t].b;
        D.s[t] = static_cast<int>(P.st[t].s);
        int sl = 0;
        while ((int64_t(1) << sl) < P.st[t].s) ++sl;
        D.sl[t] = sl;
        D.kpad[t] = P.st[t].kpad;
        D.had[t] = P.st[t].had;
        D.gfwd[t] = P.st[t].gfwd;
    }
    D.signs = P.signs;
    D.rows = rows;
    D.in = in;
    D.in_bf16 = in_dtype == HARP_BF16 ? 1 : 0;
    D.out_f32 = rotated_out;
    D.codes = codes;
    D.scales = scales;
    D.chunk = g.chunk;
    D.fuse0 = (P.st[0].b <= 8 && !P.st[0].had) ? 1 : 0;
    D.stage_base = g.stage_base;
    D.part_base = g.part_base;
    D.lev_base = g.lev_base;
    D.bar_base = g.bar_base;
    const int64_t ntiles = (rows + g.R - 1) / g.R;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ntiles, nsm[dev]));
    rows_kernel<<<grid, RT_THREADS, g.smem, static_cast<cudaStream_t>(stream)>>>(D, q, bins_exact(q, 64) ? 1 : 0);
    return cudaGetLastError();
}

int rows_fault_status(unsigned *flags) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_rows_fault, sizeof(v));
    if (e == cudaSuccess && v) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_rows_fault, &zero, sizeof(zero));
    }
    *flags = v;
    return e;
}

}  // namespace harp
