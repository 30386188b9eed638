// harp_pass.cu -- pass kernels of libharp (sm_100a): the two-sided HARP
// processor W' = M_L W M_R^T fused with the group-wise quantizer, and its
// inverse, as a short sequence of tiled passes over the matrix.
//
// What they compute:
//  * HARP (gist.science paper 2605.29843) section 2.1: each processor is a
//    product of stride stages; stage t applies one b_t x b_t block to every
//    group of coordinates {h b s + k s + l : k < b} (s = product of the later
//    radices); sections 3 and 5: two-sided on weights, inverse by the
//    transposes in reverse order. The left and right processors act on
//    different indices of W, so their stages commute with each other.
//  * PolarQuant (gist.science paper 2603.29078) sections 1 and 2: per-group
//    scale (RMS for Lloyd-Max, absmax/qmax for absmax), fp16 scale, code by
//    threshold count or rounding, and the dequantisation s * level[code].
//
// Design (B200). Every stage mixes one digit of the row index (left) or of
// the column index (right). A pass takes a run of consecutive stages of each
// side and works on tiles that are boxes in digit space: all values of the
// mixed digits, plus a short range of the neighbouring digit so that memory
// runs are contiguous and every block coefficient is reused across many
// vectors (tile columns for left stages, tile rows for right stages). A tile
// (<= 16K fp32) and the block coefficients it needs live in shared memory;
// two 256-thread CTAs share an SM so one loads while the other computes.
// Loads are cp.async (no register staging, many in flight); each stage is a
// batch of small products computed with FFMA by lanes that share a block
// (broadcast coefficient loads) and own 4 vectors x 16 outputs each, written
// back in place. Passes update an fp32 workspace in place; the first pass
// reads the input (with the sign vectors), the last one quantises and packs
// (forward) or writes the output (inverse, with the sign vectors).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <vector>

#include "harp_internal.h"
#include "harp_quant_dev.cuh"

namespace harp {
namespace {

using namespace dq;

constexpr int PT = 256;               // threads per CTA
constexpr int PW = PT / 32;           // warps per CTA
constexpr int MAXPS = 12;             // stages (both sides) in one pass
constexpr int TILE_MAX = 16384;       // tile elements
constexpr int SMEM_BUDGET = 112 * 1024;  // bytes per CTA: two CTAs per SM
constexpr int GPAD = 4;               // floats between coefficient slots

// One axis of a tile box. Global index of tile-local index i (tile position
// hb, lb): (hb*Hx + hh)*P*S + mid*S + lb*Lx + ll with hh = i / (P*Lx),
// mid = (i / Lx) % P, ll = i % Lx.
struct PAxis {
    int64_t n;        // axis length
    int64_t S;        // stride of the lowest mixed digit (1 when the pass has no stage here or ends this side)
    int P;            // product of the mixed radices (1 when none)
    int Hx, Lx;       // hi range and lo range of one tile (one of them is 1)
    int E;            // Hx * P * Lx
    int64_t nlo;      // S / Lx
    int64_t nt;       // tile positions along the axis
    const float *sign;  // sign vector applied on this axis (nullptr: none)
};

struct PStage {
    int axis;         // 0: rows (left processor), 1: cols (right)
    int b, jpad, kp;  // radix, padded inputs, padded outputs
    int sig;          // tile-local stride of the digit
    int G;            // groups in a tile
    int LV;           // lanes along vectors (32 / LV groups per warp)
    int coff;         // first coefficient slot (floats into the coefficient area)
    int gstride;      // floats per slot
    int64_t s;        // global stride of the digit
    const float *coef;  // [d/b][jpad][kp]
};

struct PassDesc {
    PAxis ax[2];
    int nst;
    PStage st[MAXPS];
    int TCp;            // tile pitch in floats (odd)
    int coef_base;      // float offset of the coefficient area
    int coef_floats;
    int tab_base;       // float offset of the index tables (rows, then cols)
    int stage_base;     // float offset of the code staging area (codes prologue)
    int smem_bytes;
    int sign_at_store;  // inverse: signs after the stages
    const void *in;
    int64_t ld_in;
    const uint8_t *in_codes;
    const uint16_t *in_scales;
    void *out;
    int64_t ld_out;
    float *out_f32;     // EPI_QUANT_F32: fp32 copy of the rotated matrix
    uint8_t *codes;
    uint16_t *scales;
    int64_t cols;       // matrix columns (row strides of codes, scales, copy)
};

__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem));
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

__host__ __device__ __forceinline__ int axis_global(const PAxis &A, int64_t pos, int i) {
    const int64_t hb = pos / A.nlo, lb = pos - hb * A.nlo;
    const int pl = A.P * A.Lx;
    const int hh = i / pl, rem = i - hh * pl;
    const int mid = rem / A.Lx, ll = rem - mid * A.Lx;
    return static_cast<int>((hb * A.Hx + hh) * A.P * A.S + mid * A.S + lb * A.Lx + ll);
}

// Global group index (c = h*s + l) of tile group gi of stage S.
__host__ __device__ __forceinline__ int64_t global_group(const PStage &S, const int *tab, int gi) {
    const int base = (gi / S.sig) * (S.b * S.sig) + gi % S.sig;
    const int64_t i = tab[base];
    const int64_t bs = static_cast<int64_t>(S.b) * S.s;
    const int64_t h = i / bs;
    return h * S.s + (i - h * bs) % S.s;
}

// ------------------------------------------------------------ one stage

// Tile addresses of one lane's 4 vectors of group gi (inputs j = 0 at p[v]),
// and its coefficient slot. Lanes past the last group or vector are clamped
// onto valid data and store nothing.
__device__ __forceinline__ void unit_addr(const PStage &S, int gi, int v0, int LV, int NV, int A, int Bv,
                                          const float *Cs, int (&p)[4], bool (&vok)[4], bool &gok,
                                          const float *&wp) {
    gok = gi < S.G;
    const int g = gok ? gi : S.G - 1;
    const int base = (g / S.sig) * (S.b * S.sig) + g % S.sig;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const int vi = v0 + LV * v;
        vok[v] = vi < NV;
        p[v] = base * A + min(vi, NV - 1) * Bv;
    }
    wp = Cs + g * S.gstride;
}

// acc[k][v] = sum_j w[j][k] * x_v[j] for K outputs and 4 vectors. Inputs
// past b are read at b-1 and meet zero coefficients.
template <int K>
__device__ __forceinline__ void unit_compute(const float *T, const float *wp, int kp, int jpad, int b,
                                             int step, const int (&p)[4], float (&acc)[K][4]) {
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[k][v] = 0.0f;
    for (int j0 = 0; j0 < jpad; j0 += 4) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int j = j0 + jj;
            const int off = min(j, b - 1) * step;
            float x[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) x[v] = T[p[v] + off];
            const float4 *w4 = reinterpret_cast<const float4 *>(wp + j * kp);
#pragma unroll
            for (int q = 0; q < K / 4; ++q) {
                const float4 w = w4[q];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    acc[4 * q + 0][v] = fmaf(w.x, x[v], acc[4 * q + 0][v]);
                    acc[4 * q + 1][v] = fmaf(w.y, x[v], acc[4 * q + 1][v]);
                    acc[4 * q + 2][v] = fmaf(w.z, x[v], acc[4 * q + 2][v]);
                    acc[4 * q + 3][v] = fmaf(w.w, x[v], acc[4 * q + 3][v]);
                }
            }
        }
    }
}

template <int K>
__device__ __forceinline__ void unit_store(float *T, int b, int k0, int step, const int (&p)[4],
                                           const bool (&vok)[4], bool gok, const float (&acc)[K][4]) {
    if (!gok) return;
#pragma unroll
    for (int k = 0; k < K; ++k) {
        if (k0 + k < b) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
                if (vok[v]) T[p[v] + (k0 + k) * step] = acc[k][v];
        }
    }
}

// One stage over the whole tile. A / Bv: tile address steps along the
// group axis / the vector axis; NV: vectors. Work units are (block of 32/LV
// groups, 4*LV vectors); with b <= 16 (one chunk of K outputs) every unit
// reads and writes only its own elements, so units update the tile in place
// without barriers. Wider blocks (ROUNDS) split the outputs into chunks of K
// over several warps, which first all read (compute into registers), then
// all write; the warps of one round hold whole (group block, vector block)s.
template <int K, bool ROUNDS>
__device__ __forceinline__ void stage_run(float *T, const float *C, const PStage &S, int A, int Bv, int NV,
                                          int warp, int lane) {
    const int LV = S.LV, LG = 32 / LV;
    const int lv = lane & (LV - 1), lg = lane / LV;
    const int span = LV * 4;
    const int nvc = (NV + span - 1) / span;
    const int ngb = (S.G + LG - 1) / LG;
    const int nkc = S.kp / K;
    const int step = S.sig * A;
    const float *Cs = C + S.coff;
    if constexpr (!ROUNDS) {
        const int nunits = ngb * nvc;
        for (int u = warp; u < nunits; u += PW) {
            const int gb = u / nvc, vc = u - gb * nvc;
            int p[4];
            bool vok[4], gok;
            const float *wp;
            unit_addr(S, gb * LG + lg, vc * span + lv, LV, NV, A, Bv, Cs, p, vok, gok, wp);
            float acc[K][4];
            unit_compute<K>(T, wp, S.kp, S.jpad, S.b, step, p, acc);
            unit_store<K>(T, S.b, 0, step, p, vok, gok, acc);
        }
    } else {
        const int nblk = ngb * nvc;
        const int bpr = PW / nkc;
        const int nrounds = (nblk + bpr - 1) / bpr;
        for (int r = 0; r < nrounds; ++r) {
            const int blk = r * bpr + warp / nkc, kc = warp - (warp / nkc) * nkc;
            const bool active = (warp < bpr * nkc) && (blk < nblk);
            float acc[K][4];
            int p[4] = {0, 0, 0, 0};
            bool vok[4] = {false, false, false, false}, gok = false;
            if (active) {
                const int gb = blk / nvc, vc = blk - gb * nvc;
                const float *wp;
                unit_addr(S, gb * LG + lg, vc * span + lv, LV, NV, A, Bv, Cs, p, vok, gok, wp);
                unit_compute<K>(T, wp + kc * K, S.kp, S.jpad, S.b, step, p, acc);
            }
            __syncthreads();
            if (active) unit_store<K>(T, S.b, kc * K, step, p, vok, gok, acc);
            __syncthreads();
        }
    }
}

// ------------------------------------------------------------ prologue / epilogue

constexpr int MAXQ = 16;   // bf16 pairs per lane when a tile row is expanded (Ec <= 1024)

// Forward-side sign factors of tile row tr / column tc (1 when none).
__device__ __forceinline__ float row_sign(const PassDesc &D, const int *rtab, int tr) {
    return D.ax[0].sign ? __ldg(D.ax[0].sign + rtab[tr]) : 1.0f;
}
__device__ __forceinline__ float col_sign(const PassDesc &D, const int *ctab, int tc) {
    return D.ax[1].sign ? __ldg(D.ax[1].sign + ctab[tc]) : 1.0f;
}

// Codes -> values for the first inverse pass: the packed words of the tile
// (staged in shared memory) and its scales; 32 codes of one row per warp step.
template <int BITS>
__device__ __forceinline__ void decode_tile(float *T, const PassDesc &D, const QuantDev &Q, const uint32_t *cw,
                                            const float *ssc, const float *lev, int warp, int lane) {
    constexpr unsigned MASK = (1u << BITS) - 1u;
    const int Er = D.ax[0].E, Ec = D.ax[1].E, TCp = D.TCp;
    const int nch = Ec >> 5, wpr = nch * BITS, ngt = Ec / Q.group;
    const int bit = lane * BITS, wi = bit >> 5, sh = bit & 31;
    for (int u = warp; u < Er * nch; u += PW) {
        const int tr = u / nch, ch = u - tr * nch;
        const unsigned w = (lane < BITS) ? cw[tr * wpr + ch * BITS + lane] : 0u;
        const unsigned w0 = __shfl_sync(FULL, w, wi);
        const unsigned w1 = __shfl_sync(FULL, w, min(wi + 1, BITS - 1));
        unsigned code = w0 >> sh;
        if (sh + BITS > 32) code |= w1 << (32 - sh);
        const float s = ssc[tr * ngt + (ch * 32) / Q.group];
        T[tr * TCp + ch * 32 + lane] = s * lev[code & MASK];
    }
}

// Scale, code and pack every (row, group) of the tile (last forward pass).
template <int BITS, bool F32COPY>
__device__ __forceinline__ void quantize_tile(const float *T, const PassDesc &D, const QuantDev &Q,
                                              const int *rtab, const int *ctab, int warp, int lane) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E, TCp = D.TCp;
    const int g = Q.group, ngt = Ec / g, per = g >> 5;
    const bool is_max = (Q.kind == HARP_ABSMAX);
    float t[(1 << BITS) - 1];
#pragma unroll
    for (int k = 0; k < (1 << BITS) - 1; ++k) t[k] = Q.thr[k];
    const int64_t spr = D.cols / g;
    const int64_t wpr = D.cols * BITS / 32;
    uint32_t *cw = reinterpret_cast<uint32_t *>(D.codes);
    for (int u = warp; u < Er * ngt; u += PW) {
        const int tr = u / ngt, gq = u - tr * ngt;
        const float *rp = T + tr * TCp + gq * g;
        float st = 0.0f;
        for (int e = 0; e < per; ++e) st = combine(st, rp[lane + 32 * e], is_max);
        const float tot = warp_reduce(st, is_max);
        const unsigned short hb = group_scale_bits(tot, Q);
        const float s = __half2float(__ushort_as_half(hb));
        const float inv = (s > 0.0f) ? __frcp_rn(s) : 0.0f;
        const int64_t row = rtab[tr];
        const int64_t c0 = ctab[0] + gq * g;
        if (lane == 0) D.scales[row * spr + c0 / g] = hb;
        for (int e = 0; e < per; ++e) {
            const float x = rp[lane + 32 * e];
            const int code = code_of<BITS>(x, s, inv, !is_max, t);
            const unsigned word = pack_words<BITS>(code, lane);
            if (lane < BITS) cw[row * wpr + (c0 / 32 + e) * BITS + lane] = word;
            if constexpr (F32COPY) D.out_f32[row * D.cols + c0 + 32 * e + lane] = x;
        }
    }
}

// ------------------------------------------------------------ the kernel

template <int PRO, int EPI>
__global__ void __launch_bounds__(PT, 2)
pass_kernel(const __grid_constant__ PassDesc D, const __grid_constant__ QuantDev Q) {
    extern __shared__ float4 sm4[];
    float *sm = reinterpret_cast<float *>(sm4);
    float *T = sm;
    float *C = sm + D.coef_base;
    int *rtab = reinterpret_cast<int *>(sm + D.tab_base);
    int *ctab = rtab + D.ax[0].E;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Er = D.ax[0].E, Ec = D.ax[1].E, TCp = D.TCp;
    const int64_t pos_c = blockIdx.x % D.ax[1].nt;
    const int64_t pos_r = blockIdx.x / D.ax[1].nt;

    for (int i = tid; i < Er; i += PT) rtab[i] = axis_global(D.ax[0], pos_r, i);
    for (int i = tid; i < Ec; i += PT) ctab[i] = axis_global(D.ax[1], pos_c, i);
    __syncthreads();

    // block coefficients of every stage of the pass (one group per warp step)
    for (int u = 0; u < D.nst; ++u) {
        const PStage &S = D.st[u];
        const int cpg = S.jpad * S.kp / 4;
        const int *tab = S.axis == 0 ? rtab : ctab;
        for (int gi = warp; gi < S.G; gi += PW) {
            const int64_t c = global_group(S, tab, gi);
            const float *src = S.coef + c * (S.jpad * S.kp);
            float *dst = C + S.coff + gi * S.gstride;
            for (int o = lane; o < cpg; o += 32) cp_async16(dst + 4 * o, src + 4 * o);
        }
    }

    // the tile
    float *lev = sm + D.stage_base;                 // codes prologue: 16 levels,
    float *ssc = lev + 16;                          // the tile's scales,
    uint32_t *cw = reinterpret_cast<uint32_t *>(ssc + ((Er * (Ec / max(Q.group, 1)) + 3) & ~3));  // its words
    if constexpr (PRO == PRO_F32) {
        const float *in = static_cast<const float *>(D.in);
        for (int tr = warp; tr < Er; tr += PW) {
            const float *src = in + static_cast<int64_t>(rtab[tr]) * D.ld_in;
            float *dst = T + tr * TCp;
            for (int tc = lane; tc < Ec; tc += 32) cp_async4(dst + tc, src + ctab[tc]);
        }
    } else if constexpr (PRO == PRO_BF16) {
        // raw bf16 pairs into the upper half of each tile row, expanded below
        const int half = Ec >> 1;
        const unsigned short *in = static_cast<const unsigned short *>(D.in);
        for (int tr = warp; tr < Er; tr += PW) {
            const unsigned short *src = in + static_cast<int64_t>(rtab[tr]) * D.ld_in;
            float *dst = T + tr * TCp + half;
            for (int q = lane; q < half; q += 32) cp_async4(dst + q, src + ctab[2 * q]);
        }
    } else {
        const int nch = Ec >> 5, wpr = nch * Q.bits, ngt = Ec / Q.group;
        const int64_t rw = D.cols * Q.bits / 32;
        const uint32_t *words = reinterpret_cast<const uint32_t *>(D.in_codes);
        for (int tr = warp; tr < Er; tr += PW) {
            const uint32_t *src = words + static_cast<int64_t>(rtab[tr]) * rw + (ctab[0] >> 5) * Q.bits;
            for (int w = lane; w < wpr; w += 32) cp_async4(cw + tr * wpr + w, src + w);
        }
        const int64_t spr = D.cols / Q.group;
        for (int i = tid; i < Er * ngt; i += PT) {
            const int tr = i / ngt, q = i - tr * ngt;
            ssc[i] = __half2float(__ushort_as_half(
                __ldg(D.in_scales + static_cast<int64_t>(rtab[tr]) * spr + ctab[0] / Q.group + q)));
        }
        if (tid < 16) lev[tid] = Q.level[tid];
    }
    cp_async_wait_all();
    __syncthreads();

    if constexpr (PRO == PRO_BF16) {
        const int half = Ec >> 1;
        for (int tr = warp; tr < Er; tr += PW) {
            float *row = T + tr * TCp;
            const float rs = D.sign_at_store ? 1.0f : row_sign(D, rtab, tr);
            unsigned w[MAXQ];
#pragma unroll
            for (int k = 0; k < MAXQ; ++k) {
                const int q = lane + 32 * k;
                w[k] = (q < half) ? __float_as_uint(row[half + q]) : 0u;
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < MAXQ; ++k) {
                const int q = lane + 32 * k;
                if (q < half) {
                    float c0 = rs, c1 = rs;
                    if (!D.sign_at_store && D.ax[1].sign) {
                        c0 *= col_sign(D, ctab, 2 * q);
                        c1 *= col_sign(D, ctab, 2 * q + 1);
                    }
                    row[2 * q] = __uint_as_float(w[k] << 16) * c0;
                    row[2 * q + 1] = __uint_as_float(w[k] & 0xffff0000u) * c1;
                }
            }
        }
        __syncthreads();
    } else if constexpr (PRO == PRO_F32) {
        if (!D.sign_at_store && (D.ax[0].sign || D.ax[1].sign)) {
            for (int tr = warp; tr < Er; tr += PW) {
                const float rs = row_sign(D, rtab, tr);
                for (int tc = lane; tc < Ec; tc += 32) T[tr * TCp + tc] *= rs * col_sign(D, ctab, tc);
            }
            __syncthreads();
        }
    } else {
        if (Q.bits == 2) decode_tile<2>(T, D, Q, cw, ssc, lev, warp, lane);
        else if (Q.bits == 3) decode_tile<3>(T, D, Q, cw, ssc, lev, warp, lane);
        else decode_tile<4>(T, D, Q, cw, ssc, lev, warp, lane);
        __syncthreads();
    }

    // the stages
    for (int u = 0; u < D.nst; ++u) {
        const PStage &S = D.st[u];
        const bool rows = (S.axis == 0);
        const int A = rows ? TCp : 1, Bv = rows ? 1 : TCp, NV = rows ? Ec : Er;
        if (S.kp == 8) stage_run<8, false>(T, C, S, A, Bv, NV, warp, lane);
        else if (S.kp == 16) stage_run<16, false>(T, C, S, A, Bv, NV, warp, lane);
        else stage_run<8, true>(T, C, S, A, Bv, NV, warp, lane);
        __syncthreads();
    }

    // epilogue
    if constexpr (EPI == EPI_QUANT || EPI == EPI_QUANT_F32) {
        constexpr bool F = (EPI == EPI_QUANT_F32);
        if (Q.bits == 2) quantize_tile<2, F>(T, D, Q, rtab, ctab, warp, lane);
        else if (Q.bits == 3) quantize_tile<3, F>(T, D, Q, rtab, ctab, warp, lane);
        else quantize_tile<4, F>(T, D, Q, rtab, ctab, warp, lane);
    } else {
        const bool sg = D.sign_at_store && (D.ax[0].sign || D.ax[1].sign);
        for (int tr = warp; tr < Er; tr += PW) {
            const int64_t ro = static_cast<int64_t>(rtab[tr]) * D.ld_out;
            const float rs = sg ? row_sign(D, rtab, tr) : 1.0f;
            for (int tc = lane; tc < Ec; tc += 32) {
                float v = T[tr * TCp + tc];
                if (sg) v *= rs * col_sign(D, ctab, tc);
                if constexpr (EPI == EPI_BF16)
                    static_cast<__nv_bfloat16 *>(D.out)[ro + ctab[tc]] = __float2bfloat16_rn(v);
                else
                    static_cast<float *>(D.out)[ro + ctab[tc]] = v;
            }
        }
    }
}

}  // namespace

// ------------------------------------------------------------ host: planning

namespace {

struct AxisGeo {
    int P;
    int64_t S;
};

AxisGeo axis_geo(const PlanDev *pl, int i, int j) {
    if (!pl || i == j) return {1, 1};
    int64_t p = 1;
    for (int t = i; t < j; ++t) p *= pl->st[t].b;
    return {static_cast<int>(p), pl->st[j - 1].s};
}

// Divisors of n not above lim, ascending.
void divisors(int64_t n, int64_t lim, std::vector<int> &out) {
    out.clear();
    std::vector<int> hi;
    for (int64_t a = 1; a * a <= n && a <= lim; ++a) {
        if (n % a) continue;
        out.push_back(static_cast<int>(a));
        const int64_t b = n / a;
        if (b != a && b <= lim) hi.push_back(static_cast<int>(b));
    }
    for (auto it = hi.rbegin(); it != hi.rend(); ++it) out.push_back(*it);
}

// Lanes along the vectors for a stage with G groups and NV vectors: the
// power of two in [1, 32] that wastes the fewest lane slots (ties: more
// lanes along the vectors).
int pick_lv(int G, int NV) {
    int best = 32;
    double bu = -1.0;
    for (int lv = 32; lv >= 1; lv >>= 1) {
        const int lg = 32 / lv;
        const int64_t vs = static_cast<int64_t>(lv) * 4 * ((NV + lv * 4 - 1) / (lv * 4));
        const int64_t gs = static_cast<int64_t>(lg) * ((G + lg - 1) / lg);
        const double u = static_cast<double>(NV) / vs * static_cast<double>(G) / gs;
        if (u > bu + 1e-9) { bu = u; best = lv; }
    }
    return best;
}

struct Cand {
    bool ok = false;
    int XL = 0, XR = 0;
    double score = 0.0;
};

struct PlanInput {
    const PlanDev *L;   // may be null (right-only)
    const PlanDev *R;
    int64_t rows, cols;
    int group;
};

int stage_coef_floats(const PlanDev *pl, int i, int j, int E) {
    int f = 0;
    for (int t = i; t < j; ++t) {
        const StageDev &s = pl->st[t];
        f += (E / s.b) * (s.jpad * s.kp + GPAD);
    }
    return f;
}

int tcp_of(int Ec) { return (Ec % 2 == 0) ? Ec + 1 : Ec; }

// Shared-memory bytes of a tile (layout of PassDesc: tile, coefficients,
// tables, code staging).
int64_t tile_smem(const PlanInput &in, int iL, int jL, int iR, int jR, int Er, int Ec, bool codes_stage) {
    int64_t f = (static_cast<int64_t>(Er) * tcp_of(Ec) + 3) & ~int64_t(3);
    if (in.L) f += stage_coef_floats(in.L, iL, jL, Er);
    f += stage_coef_floats(in.R, iR, jR, Ec);
    f += Er + Ec;
    if (codes_stage) f += 16 + ((static_cast<int64_t>(Er) * (Ec / in.group) + 3) & ~int64_t(3)) +
                          static_cast<int64_t>(Er) * Ec * 4 / 32;
    return f * 4;
}

// Best tile for a pass applying L[iL:jL] and R[iR:jR]; `last` passes
// quantise (forward) / decode codes (inverse) and need whole groups of
// contiguous columns; `first` passes may read bf16 pairs.
Cand best_tile(const PlanInput &in, int iL, int jL, int iR, int jR, bool first, bool last) {
    Cand best;
    const AxisGeo gl = axis_geo(in.L, iL, jL), gr = axis_geo(in.R, iR, jR);
    const bool hasL = in.L && jL > iL, hasR = jR > iR;
    const int64_t nl = (gl.S > 1) ? gl.S : in.rows / gl.P;
    const int64_t nr = (gr.S > 1) ? gr.S : in.cols / gr.P;
    std::vector<int> xl, xr;
    divisors(nl, TILE_MAX / std::max(gl.P, 1), xl);
    divisors(nr, TILE_MAX / std::max(gr.P, 1), xr);
    for (int XL : xl) {
        const int64_t Er = static_cast<int64_t>(gl.P) * XL;
        if (Er > TILE_MAX) break;
        for (int XR : xr) {
            const int64_t Ec = static_cast<int64_t>(gr.P) * XR;
            if (Er * Ec > TILE_MAX) break;
            const int64_t run = (gr.S > 1) ? XR : Ec;       // contiguous columns in memory
            if (run % 2) continue;                          // bf16 pairs, 8-byte f32 pairs
            if (last && (Ec % in.group || Ec % 32)) continue;
            if (first && Ec > 2 * 32 * MAXQ) continue;
            if (tile_smem(in, iL, jL, iR, jR, static_cast<int>(Er), static_cast<int>(Ec), last) > SMEM_BUDGET)
                continue;
            int64_t nv = TILE_MAX;
            if (hasL) nv = std::min<int64_t>(nv, Ec);
            if (hasR) nv = std::min<int64_t>(nv, Er);
            const double sc = std::min<int64_t>(nv, 128) * 1000.0 + std::min<int64_t>(run, 16) * 10.0 +
                              static_cast<double>(Er * Ec) / 2048.0;
            if (!best.ok || sc > best.score) {
                best.ok = true;
                best.XL = XL;
                best.XR = XR;
                best.score = sc;
            }
        }
    }
    return best;
}

struct PassSpec {
    int iL, jL, iR, jR, XL, XR;
};

// Fewest passes (then best summed tile score) that take both processors
// from stage 0 to the end; each pass takes a run of the next stages of
// either side (at most MAXPS in all).
bool plan_passes(const PlanInput &in, std::vector<PassSpec> &out) {
    const int mL = in.L ? in.L->m : 0, mR = in.R->m;
    const int W = mR + 1;
    const int NS = (mL + 1) * W;
    const int INF = 1 << 20;
    std::vector<int> npass(NS, INF);
    std::vector<double> score(NS, -1.0);
    std::vector<PassSpec> next(NS);
    npass[mL * W + mR] = 0;
    score[mL * W + mR] = 0.0;
    for (int iL = mL; iL >= 0; --iL) {
        for (int iR = mR; iR >= 0; --iR) {
            if (iL == mL && iR == mR) continue;
            const int id = iL * W + iR;
            for (int jL = iL; jL <= mL; ++jL) {
                for (int jR = iR; jR <= mR; ++jR) {
                    if (jL == iL && jR == iR) continue;
                    if ((jL - iL) + (jR - iR) > MAXPS) continue;
                    const int nid = jL * W + jR;
                    if (npass[nid] >= INF) continue;
                    const bool last = (jL == mL && jR == mR);
                    const Cand c = best_tile(in, iL, jL, iR, jR, iL == 0 && iR == 0, last);
                    if (!c.ok) continue;
                    const int np = npass[nid] + 1;
                    const double sc = score[nid] + c.score;
                    if (np < npass[id] || (np == npass[id] && sc > score[id])) {
                        npass[id] = np;
                        score[id] = sc;
                        next[id] = PassSpec{iL, jL, iR, jR, c.XL, c.XR};
                    }
                }
            }
        }
    }
    if (npass[0] >= INF) return false;
    out.clear();
    int id = 0;
    while (id != mL * W + mR) {
        out.push_back(next[id]);
        id = next[id].jL * W + next[id].jR;
    }
    return true;
}

void fill_axis(PAxis &A, const PlanDev *pl, int i, int j, int X, int64_t n) {
    const AxisGeo g = axis_geo(pl, i, j);
    A.n = n;
    A.P = g.P;
    A.S = g.S;
    if (g.S > 1) { A.Hx = 1; A.Lx = X; } else { A.Hx = X; A.Lx = 1; }
    A.E = A.Hx * A.P * A.Lx;
    A.nlo = g.S / A.Lx;
    A.nt = (n / (static_cast<int64_t>(A.P) * g.S * A.Hx)) * A.nlo;
    A.sign = nullptr;
}

// Stage descriptors of a pass: forward applies L[iL..jL) then R[iR..jR) in
// ascending order; inverse applies R[jR-1..iR] then L[jL-1..iL] with the
// transposed blocks.
void fill_stages(PassDesc &D, const PlanInput &in, const PassSpec &ps, bool inverse, int &coef_floats) {
    struct Ref { int axis, t; };
    Ref refs[2 * HARP_MAX_STAGES];
    int n = 0;
    if (!inverse) {
        for (int t = ps.iL; t < ps.jL; ++t) refs[n++] = {0, t};
        for (int t = ps.iR; t < ps.jR; ++t) refs[n++] = {1, t};
    } else {
        for (int t = ps.jR - 1; t >= ps.iR; --t) refs[n++] = {1, t};
        for (int t = ps.jL - 1; t >= ps.iL; --t) refs[n++] = {0, t};
    }
    D.nst = n;
    coef_floats = 0;
    for (int u = 0; u < n; ++u) {
        const PlanDev *pl = refs[u].axis == 0 ? in.L : in.R;
        const int t = refs[u].t;
        const int jEnd = refs[u].axis == 0 ? ps.jL : ps.jR;
        const PAxis &A = D.ax[refs[u].axis];
        const StageDev &sd = pl->st[t];
        int64_t sig = 1;
        for (int v = t + 1; v < jEnd; ++v) sig *= pl->st[v].b;
        PStage &S = D.st[u];
        S.axis = refs[u].axis;
        S.b = sd.b;
        S.jpad = sd.jpad;
        S.kp = sd.kp;
        S.sig = static_cast<int>(sig) * A.Lx;
        S.G = A.E / sd.b;
        S.LV = pick_lv(S.G, refs[u].axis == 0 ? D.ax[1].E : D.ax[0].E);
        S.coff = coef_floats;
        S.gstride = sd.jpad * sd.kp + GPAD;
        S.s = sd.s;
        S.coef = inverse ? sd.pinv : sd.pfwd;
        coef_floats += S.G * S.gstride;
    }
}

template <int PRO, int EPI>
int launch_pass(const PassDesc &D, const QuantDev &Q, cudaStream_t st) {
    static int attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && attr_done[dev] < D.smem_bytes) {
        const cudaError_t e = cudaFuncSetAttribute(pass_kernel<PRO, EPI>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BUDGET);
        if (e != cudaSuccess) return e;
        attr_done[dev] = SMEM_BUDGET;
    }
    const int64_t nb = D.ax[0].nt * D.ax[1].nt;
    if (nb <= 0) return 0;
    pass_kernel<PRO, EPI><<<static_cast<unsigned>(nb), PT, D.smem_bytes, st>>>(D, Q);
    return cudaGetLastError();
}

int dispatch(const PassDesc &D, const QuantDev &Q, int pro, int epi, cudaStream_t st) {
    switch (pro * 4 + epi) {
        case PRO_F32 * 4 + EPI_F32: return launch_pass<PRO_F32, EPI_F32>(D, Q, st);
        case PRO_F32 * 4 + EPI_BF16: return launch_pass<PRO_F32, EPI_BF16>(D, Q, st);
        case PRO_F32 * 4 + EPI_QUANT: return launch_pass<PRO_F32, EPI_QUANT>(D, Q, st);
        case PRO_F32 * 4 + EPI_QUANT_F32: return launch_pass<PRO_F32, EPI_QUANT_F32>(D, Q, st);
        case PRO_BF16 * 4 + EPI_F32: return launch_pass<PRO_BF16, EPI_F32>(D, Q, st);
        case PRO_BF16 * 4 + EPI_QUANT: return launch_pass<PRO_BF16, EPI_QUANT>(D, Q, st);
        case PRO_BF16 * 4 + EPI_QUANT_F32: return launch_pass<PRO_BF16, EPI_QUANT_F32>(D, Q, st);
        case PRO_CODES * 4 + EPI_F32: return launch_pass<PRO_CODES, EPI_F32>(D, Q, st);
        case PRO_CODES * 4 + EPI_BF16: return launch_pass<PRO_CODES, EPI_BF16>(D, Q, st);
        default: return cudaErrorInvalidValue;
    }
}

// Build the descriptor of pass k of a plan (geometry, stages, shared-memory
// layout); prologue/epilogue pointers are filled by the caller.
void build_desc(PassDesc &D, const PlanInput &in, const PassSpec &ps, bool inverse, bool codes_stage) {
    D = PassDesc{};
    fill_axis(D.ax[0], in.L, ps.iL, ps.jL, ps.XL, in.rows);
    fill_axis(D.ax[1], in.R, ps.iR, ps.jR, ps.XR, in.cols);
    int cf = 0;
    fill_stages(D, in, ps, inverse, cf);
    D.TCp = tcp_of(D.ax[1].E);
    D.coef_base = (D.ax[0].E * D.TCp + 3) & ~3;
    D.coef_floats = cf;
    D.tab_base = D.coef_base + cf;
    D.stage_base = D.tab_base + D.ax[0].E + D.ax[1].E;
    int64_t total = D.stage_base;
    if (codes_stage)
        total += 16 + ((static_cast<int64_t>(D.ax[0].E) * (D.ax[1].E / in.group) + 3) & ~int64_t(3)) +
                 static_cast<int64_t>(D.ax[0].E) * D.ax[1].E * 4 / 32;
    D.smem_bytes = static_cast<int>(total * 4);
    if (in.L && ps.iL == 0 && ps.jL > 0) D.ax[0].sign = in.L->signs;
    if (ps.iR == 0 && ps.jR > 0) D.ax[1].sign = in.R->signs;
    D.sign_at_store = inverse ? 1 : 0;
    D.cols = in.cols;
}

}  // namespace

bool pass_plan_ok(const PlanDev &left, const PlanDev &right, int group) {
    PlanInput in{&left, &right, left.d, right.d, group};
    std::vector<PassSpec> ps;
    return plan_passes(in, ps);
}

int launch_pass_fwd(const PlanDev &left, const PlanDev &right, const QuantDev &q, const void *in_ptr,
                    int in_dtype, uint8_t *codes, uint16_t *scales, float *rotated_out, float *ws,
                    void *stream) {
    PlanInput in{&left, &right, left.d, right.d, q.group};
    std::vector<PassSpec> ps;
    if (!plan_passes(in, ps)) return cudaErrorInvalidValue;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int np = static_cast<int>(ps.size());
    for (int k = 0; k < np; ++k) {
        const bool first = (k == 0), last = (k == np - 1);
        PassDesc D;
        build_desc(D, in, ps[k], false, last);
        int pro = PRO_F32, epi = EPI_F32;
        if (first) {
            pro = (in_dtype == HARP_BF16) ? PRO_BF16 : PRO_F32;
            D.in = in_ptr;
        } else {
            D.in = ws;
        }
        D.ld_in = in.cols;
        if (last) {
            epi = rotated_out ? EPI_QUANT_F32 : EPI_QUANT;
            D.codes = codes;
            D.scales = scales;
            D.out_f32 = rotated_out;
        } else {
            D.out = ws;
            D.ld_out = in.cols;
        }
        const int e = dispatch(D, q, pro, epi, st);
        if (e) return e;
    }
    return 0;
}

int launch_pass_inv(const PlanDev &left, const PlanDev &right, const QuantDev &q, const uint8_t *codes,
                    const uint16_t *scales, void *out, int out_dtype, float *ws, void *stream) {
    PlanInput in{&left, &right, left.d, right.d, q.group};
    std::vector<PassSpec> ps;
    if (!plan_passes(in, ps)) return cudaErrorInvalidValue;
    std::reverse(ps.begin(), ps.end());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int np = static_cast<int>(ps.size());
    for (int k = 0; k < np; ++k) {
        const bool first = (k == 0), last = (k == np - 1);
        PassDesc D;
        build_desc(D, in, ps[k], true, first);
        int pro = PRO_F32, epi = EPI_F32;
        if (first) {
            pro = PRO_CODES;
            D.in_codes = codes;
            D.in_scales = scales;
        } else {
            D.in = ws;
            D.ld_in = in.cols;
        }
        D.ld_out = in.cols;
        if (last) {
            epi = (out_dtype == HARP_BF16) ? EPI_BF16 : EPI_F32;
            D.out = out;
        } else {
            D.out = ws;
        }
        const int e = dispatch(D, q, pro, epi, st);
        if (e) return e;
    }
    return 0;
}

}  // namespace harp
