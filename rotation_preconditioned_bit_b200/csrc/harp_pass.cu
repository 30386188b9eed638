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
#include "harp_tc.cuh"

namespace harp {
namespace {

using namespace dq;

constexpr int PT = 512;               // threads per CTA (one CTA per SM)
constexpr int PW = PT / 32;           // warps per CTA
constexpr int MAXPS = 12;             // stages (both sides) in one pass
constexpr int TILE_MAX = 16384;       // tile elements
constexpr int SMEM_BUDGET = 232448;    // bytes per CTA (opt-in maximum): two tile buffers
constexpr int GPAD = 4;               // floats between coefficient slots
constexpr int TC_MIN_SMEM = 120 * 1024;
constexpr int MAX_SLOTS_HOST = 8;     // tensor-core slots at the narrowest blocks (512 / 64)  // shared memory of a tensor-core CTA: more than half an SM's

// Division by a fixed divisor d >= 1 as a multiply-high and a shift (exact
// for dividends below 2^31): sh = ceil(log2 d), mul = 2^32 (2^sh - d) / d + 1.
struct FDiv {
    unsigned d, mul;
    int sh;
};

inline FDiv make_fdiv(unsigned d) {
    FDiv f;
    f.d = d;
    f.sh = 0;
    while ((1u << f.sh) < d) ++f.sh;
    f.mul = static_cast<unsigned>(((uint64_t(1) << 32) * ((uint64_t(1) << f.sh) - d)) / d + 1);
    return f;
}

__host__ __device__ __forceinline__ unsigned fdiv(unsigned u, const FDiv &f) {
#ifdef __CUDA_ARCH__
    return (__umulhi(u, f.mul) + u) >> f.sh;
#else
    return static_cast<unsigned>((((static_cast<uint64_t>(u) * f.mul) >> 32) + u) >> f.sh);
#endif
}

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
    FDiv f_nlo, f_PS, f_S, f_Hx, f_Lx;   // divisions by nlo, P*S, S, Hx, Lx
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
    int had;          // every block is the normalised Sylvester Hadamard: butterfly, no coefficients
    // tensor-core stages (the tcgen05 build): the stage as a batch of
    // split-precision products, one MMA "instance" per (group, block of mb
    // vectors): D[v][k] = sum_j x_v[j] B[k][j], K = N = up.
    int up;           // b rounded up to 16
    int mb;           // vectors per instance: 128, or 64 (two instances share TMEM columns)
    int nvb;          // vector blocks of mb
    int nslots;       // TMEM slots of 4*up columns (A hi, A lo, D)
    int ucoff;        // byte offset of the stage's operand blocks in the coefficient area
    const float *ucoef; // [d/b][2 up up] operand blocks (forward or inverse)
    FDiv f_nvb, f_sig;  // divisions by nvb and sig
};

struct PassDesc {
    PAxis ax[2];
    int nst;
    PStage st[MAXPS];
    int TCp;            // tile pitch in floats (odd)
    int buf_floats;     // floats per coefficient+table buffer (two buffers follow the tile)
    int tile_floats;    // floats of the tile (first in shared memory)
    int lev_base;       // float offset of the 16 dequantised levels
    int loc_base;       // float offset of the per-pass local index tables (rows, then columns)
    FDiv f_nch;         // division by the number of 32-column chunks of a tile row
    FDiv f_wpr;         // ... by the packed code words of a tile row
    FDiv f_ngt;         // ... by the quantiser groups of a tile row
    FDiv f_gch;         // ... by the 32-code chunks of a quantiser group
    FDiv f_nq;          // ... by the column quads of a tile row
    FDiv f_nchc;        // ... by the 32-column chunks of a tile row (codes)
    FDiv f_nchc4;       // ... by the groups of 4 such chunks
    int stage_base;     // float offset of the staging buffer of the next tile's input
    int coef_base;      // float offset of the coefficient area
    int coef_floats;
    int tab_base;       // float offset of the index tables (rows, then cols)
    int coef_single;    // tensor-core build: one coefficient area at coef_base, refilled stage by stage
    int in_bulk;        // tensor-core build: 0 = cp.async, 1 = one contiguous tile (bulk copy),
                        // 2 = one bulk copy per tile row of in_row_bytes
    int in_row_bytes;
    int tc_base;        // tensor-core build: float offset of the TMEM address slot and the mbarrier
    int smem_bytes;
    int sign_at_store;  // inverse: signs after the stages
    int bins;           // quantising pass: Lloyd-Max codes by the 64-bin table (exact for these midpoints)
    int in_blocked;     // input is a workspace in this pass's tile-major layout
    int out_blocked;    // output is a workspace in the next pass's tile-major layout
    PAxis nx[2];        // the next pass's tile geometry (out_blocked)
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

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Global index along axis A of tile-local index i at tile position pos
// (32-bit: every index is below the axis length d < 2^31).
__host__ __device__ __forceinline__ int axis_global(const PAxis &A, unsigned pos, int i) {
    const unsigned nlo = static_cast<unsigned>(A.nlo), S = static_cast<unsigned>(A.S);
    const unsigned hb = pos / nlo, lb = pos - hb * nlo;
    const unsigned pl = static_cast<unsigned>(A.P * A.Lx);
    const unsigned hh = static_cast<unsigned>(i) / pl, rem = static_cast<unsigned>(i) - hh * pl;
    const unsigned mid = rem / A.Lx, ll = rem - mid * A.Lx;
    return static_cast<int>((hb * A.Hx + hh) * A.P * S + mid * S + lb * A.Lx + ll);
}

// Inverse of axis_global: tile position and tile-local index of global
// index i.
__host__ __device__ __forceinline__ void axis_local(const PAxis &A, int i, unsigned &pos, int &loc) {
    const unsigned u = static_cast<unsigned>(i);
    const unsigned hi = fdiv(u, A.f_PS), rem = u - hi * A.f_PS.d;
    const unsigned mid = fdiv(rem, A.f_S), lo = rem - mid * A.f_S.d;
    const unsigned hb = fdiv(hi, A.f_Hx), hh = hi - hb * A.Hx, lb = fdiv(lo, A.f_Lx), ll = lo - lb * A.Lx;
    pos = hb * static_cast<unsigned>(A.nlo) + lb;
    loc = static_cast<int>((hh * A.P + mid) * A.Lx + ll);
}

// Global index of the first element (local index 0) of the tile at
// position pos; local index i adds axis_global(A, 0, i) - axis_global(A, 0, 0).
__host__ __device__ __forceinline__ int axis_base(const PAxis &A, unsigned pos) {
    const unsigned hb = fdiv(pos, A.f_nlo), lb = pos - hb * static_cast<unsigned>(A.nlo);
    return static_cast<int>(hb * A.Hx * A.f_PS.d + lb * A.Lx);
}

// Global group index (c = h*s + l) of tile group gi of stage S.
__host__ __device__ __forceinline__ int global_group(const PStage &S, const int *tab, int gi) {
    const int base = (gi / S.sig) * (S.b * S.sig) + gi % S.sig;
    const unsigned i = static_cast<unsigned>(tab[base]);
    const unsigned s = static_cast<unsigned>(S.s), bs = static_cast<unsigned>(S.b) * s;
    const unsigned h = i / bs;
    return static_cast<int>(h * s + (i - h * bs) % s);
}

// ------------------------------------------------------------ one stage

// Packed fp32 pairs (two IEEE single-precision FMAs per instruction; each
// half rounds exactly like fmaf).
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

// Vectors per lane in a stage work unit.
constexpr int VL = 2;

// Tile addresses of one lane's VL vectors of group gi (inputs j = 0 at
// p[v]), and its coefficient slot. Lanes past the last group or vector are
// clamped onto valid data and store nothing.
__device__ __forceinline__ void unit_addr(const PStage &S, int gi, int v0, int LV, int NV, int A, int Bv,
                                          const float *Cs, int (&p)[VL], bool (&vok)[VL], bool &gok,
                                          const float *&wp) {
    gok = gi < S.G;
    const int g = gok ? gi : S.G - 1;
    const int base = (g / S.sig) * (S.b * S.sig) + g % S.sig;
#pragma unroll
    for (int v = 0; v < VL; ++v) {
        const int vi = v0 + LV * v;
        vok[v] = vi < NV;
        p[v] = base * A + min(vi, NV - 1) * Bv;
    }
    wp = Cs + g * S.gstride;
}

// acc[q][v] = (out 2q, out 2q+1) of vector v: sum_j w[j][k] * x_v[j] for K
// outputs and VL vectors, as packed pairs of outputs: the coefficient row
// w[j][0..K) is read as K/4 16-byte words, each two ready-made pairs, and
// x_v[j] is broadcast into both halves. CLAMP: inputs past b are read at b-1
// and meet zero coefficients (only when b is not a multiple of 4).
// EXACT: b = jpad = kp = K (fixed trip count, no clamping): the loop is
// unrolled completely.
template <int K, bool CLAMP, bool EXACT = false>
__device__ __forceinline__ void unit_compute(const float *T, const float *wp, int kp_rt, int jpad_rt, int b_rt,
                                             int step, const int (&p)[VL], f2_t (&acc)[K / 2][VL]) {
    const int kp = EXACT ? K : kp_rt, jpad = EXACT ? K : jpad_rt, b = EXACT ? K : b_rt;
#pragma unroll
    for (int q = 0; q < K / 2; ++q)
#pragma unroll
        for (int v = 0; v < VL; ++v) acc[q][v] = 0ull;
    const float *xp[VL];
#pragma unroll
    for (int v = 0; v < VL; ++v) xp[v] = T + p[v];
    const ulonglong2 *wq = reinterpret_cast<const ulonglong2 *>(wp);
    const int wstep = kp / 4;      // 16-byte words per coefficient row
    const int jlast = (b - 1) * step;
#pragma unroll(EXACT ? K : 4)
    for (int j = 0; j < jpad; ++j) {
        f2_t x[VL];
#pragma unroll
        for (int v = 0; v < VL; ++v) {
            const float xv = CLAMP ? xp[v][min(j * step, jlast)] : *xp[v];
            x[v] = f2_pack(xv, xv);
            if (!CLAMP) xp[v] += step;
        }
#pragma unroll
        for (int q = 0; q < K / 4; ++q) {
            const ulonglong2 w = wq[q];
#pragma unroll
            for (int v = 0; v < VL; ++v) {
                acc[2 * q][v] = f2_fma(w.x, x[v], acc[2 * q][v]);
                acc[2 * q + 1][v] = f2_fma(w.y, x[v], acc[2 * q + 1][v]);
            }
        }
        wq += wstep;
    }
}

template <int K>
__device__ __forceinline__ void unit_store(float *T, int b, int k0, int step, const int (&p)[VL],
                                           const bool (&vok)[VL], bool gok, const f2_t (&acc)[K / 2][VL]) {
    if (!gok) return;
#pragma unroll
    for (int v = 0; v < VL; ++v) {
        if (!vok[v]) continue;
        float *y = T + p[v] + k0 * step;
#pragma unroll
        for (int q = 0; q < K / 2; ++q) {
            float lo, hi;
            f2_unpack(acc[q][v], lo, hi);
            if (k0 + 2 * q < b) y[(2 * q) * step] = lo;
            if (k0 + 2 * q + 1 < b) y[(2 * q + 1) * step] = hi;
        }
    }
}

// One stage over the whole tile. A / Bv: tile address steps along the
// group axis / the vector axis; NV: vectors. Work units are (block of 32/LV
// groups, VL*LV vectors); with b <= 16 (one chunk of K outputs) every unit
// reads and writes only its own elements, so units update the tile in place
// without barriers. Wider blocks (ROUNDS) split the outputs into chunks of K
// over several warps, which first all read (compute into registers), then
// all write; the warps of one round hold whole (group block, vector block)s.
// EXACT (no ROUNDS): every block of the stage has b = K outputs and inputs.
template <int K, bool ROUNDS, bool EXACT = false>
__device__ __forceinline__ void stage_run(float *T, const float *C, const PStage &S, int A, int Bv, int NV,
                                          int warp, int lane) {
    const int LV = S.LV, LG = 32 / LV;
    const int lv = lane & (LV - 1), lg = lane / LV;
    const int span = LV * VL;
    const int nvc = (NV + span - 1) / span;
    const int ngb = (S.G + LG - 1) / LG;
    const int nkc = S.kp / K;
    const int step = S.sig * A;
    const bool clamp = (S.jpad != S.b);
    const float *Cs = C + S.coff;
    if constexpr (!ROUNDS) {
        const int nunits = ngb * nvc;
        for (int u = warp; u < nunits; u += PW) {
            const int gb = u / nvc, vc = u - gb * nvc;
            int p[VL];
            bool vok[VL], gok;
            const float *wp;
            unit_addr(S, gb * LG + lg, vc * span + lv, LV, NV, A, Bv, Cs, p, vok, gok, wp);
            f2_t acc[K / 2][VL];
            if constexpr (EXACT) {
                unit_compute<K, false, true>(T, wp, K, K, K, step, p, acc);
                unit_store<K>(T, K, 0, step, p, vok, gok, acc);
            } else {
                if (clamp) unit_compute<K, true>(T, wp, S.kp, S.jpad, S.b, step, p, acc);
                else unit_compute<K, false>(T, wp, S.kp, S.jpad, S.b, step, p, acc);
                unit_store<K>(T, S.b, 0, step, p, vok, gok, acc);
            }
        }
    } else {
        const int nblk = ngb * nvc;
        const int bpr = PW / nkc;
        const int nrounds = (nblk + bpr - 1) / bpr;
        for (int r = 0; r < nrounds; ++r) {
            const int blk = r * bpr + warp / nkc, kc = warp - (warp / nkc) * nkc;
            const bool active = (warp < bpr * nkc) && (blk < nblk);
            f2_t acc[K / 2][VL];
            int p[VL];
            bool vok[VL], gok = false;
#pragma unroll
            for (int v = 0; v < VL; ++v) { p[v] = 0; vok[v] = false; }
            if (active) {
                const int gb = blk / nvc, vc = blk - gb * nvc;
                const float *wp;
                unit_addr(S, gb * LG + lg, vc * span + lv, LV, NV, A, Bv, Cs, p, vok, gok, wp);
                unit_compute<K, true>(T, wp + kc * K, S.kp, S.jpad, S.b, step, p, acc);
            }
            __syncthreads();
            if (active) unit_store<K>(T, S.b, kc * K, step, p, vok, gok, acc);
            __syncthreads();
        }
    }
}

// A stage whose blocks are all the normalised Sylvester Hadamard matrix H_b
// (HARP section 2.2, theta = 0): each lane keeps the b inputs of its
// vectors in registers and applies the fast Walsh-Hadamard butterfly, log2 b
// rounds of (a + c, a - c) on pairs h apart, which computes
// sum_j (-1)^popcount(k & j) x_j for every output k, then scales by the
// block entry 1/sqrt(b). In place: every lane writes only the elements it read.
template <int B>
__device__ __forceinline__ void stage_fwht(float *T, const PStage &S, int A, int Bv, int NV, int warp, int lane) {
    const int LV = S.LV, LG = 32 / LV;
    const int lv = lane & (LV - 1), lg = lane / LV;
    const int span = LV * VL;
    const int nvc = (NV + span - 1) / span;
    const int ngb = (S.G + LG - 1) / LG;
    const int step = S.sig * A;
    const float scale = static_cast<float>(1.0 / sqrt(static_cast<double>(B)));
    for (int u = warp; u < ngb * nvc; u += PW) {
        const int gb = u / nvc, vc = u - gb * nvc;
        const int gi = gb * LG + lg;
        const bool gok = gi < S.G;
        const int g = gok ? gi : S.G - 1;
        const int base = (g / S.sig) * (S.b * S.sig) + g % S.sig;
#pragma unroll
        for (int v = 0; v < VL; ++v) {
            const int vi = vc * span + lv + LV * v;
            const bool ok = gok && vi < NV;
            float *xp = T + base * A + min(vi, NV - 1) * Bv;
            float x[B];
#pragma unroll
            for (int j = 0; j < B; ++j) x[j] = xp[j * step];
#pragma unroll
            for (int h = 1; h < B; h <<= 1)
#pragma unroll
                for (int i = 0; i < B; ++i)
                    if ((i & h) == 0) {
                        const float a = x[i], c = x[i + h];
                        x[i] = a + c;
                        x[i + h] = a - c;
                    }
            if (ok) {
#pragma unroll
                for (int j = 0; j < B; ++j) xp[j * step] = x[j] * scale;
            }
        }
    }
}

// Stages with blocks wider than 16 (rare) run out of line so that their
// barrier-separated rounds do not raise the register pressure of the rest.
__device__ __noinline__ void stage_rounds(float *T, const float *C, const PStage &S, int A, int Bv, int NV,
                                          int warp, int lane) {
    stage_run<8, true>(T, C, S, A, Bv, NV, warp, lane);
}

// ------------------------------------------------------------ tensor-core stage

// Device record of bounded waits that ran out (bit 0: an MMA batch never
// completed). Kernels never trap; the host reads this with
// harp_fault_status.
__device__ unsigned int g_pass_fault;

constexpr int TMEM_COLS = 512;
constexpr long long MMA_WAIT_LIMIT = 1ll << 30;   // SM cycles (about half a second)

// One block stage on the tensor cores (tcgen05.mma kind::tf32, 3xTF32):
// every instance (group g, block of mb vectors) is the product
//     D[v][n] = sum_j x_v[j] * Bop[n][j],   n < 2*UP,  j < UP,
// of the vectors' inputs (rows of A, in TMEM: tf32 hi in UP columns, the
// tf32 remainder lo in the next UP) and the group's operand block (2*UP rows:
// the tf32 coefficients, then their remainders; shared memory). Per 8-input
// step one MMA multiplies A_hi by all 2*UP rows (N = 2*UP) and one adds A_lo
// times the hi rows (N = UP) into the first half, so the output is
//     y_v[k] = D[v][k] + D[v][UP + k]
//            = sum_j (x_hi b_hi + x_lo b_hi) + sum_j x_hi b_lo,
// x*b to about 2^-22 relative with fp32 accumulation.
//
// TMEM (512 columns) holds SLOTS slots of 4*UP columns (A hi | A lo | D); a
// slot carries one instance (mb = 128) or two (mb = 64, lanes 0-15 and 16-31
// of every 32-lane quarter). A stage runs in rounds of up to SLOTS slots:
//   1. every warp splits and stores its items (slot, 16-column chunk) of its
//      TMEM quarter (warp w serves lanes 32*(w%4)..+31), all before one
//      tcgen05.wait::st, then arrives on each touched slot's "A full"
//      mbarrier (the 4*UP/16 items of a slot arrive with AFULL_COUNT in
//      total);
//   2. warps 0..3 (one elected thread each) take every fourth slot: wait for
//      its A, issue its MMAs, commit to its "D full" mbarrier;
//   3. every warp waits for the slots of its items, loads their D with one
//      tcgen05.wait::ld, and writes y back into the tile in place.
// The MMAs of early slots run while later slots are still being stored and
// earlier ones read back. Inputs past b are zeros, outputs past b are
// dropped. Returns false when a wait ran out (the stage is then abandoned).
constexpr int MAX_SLOTS = TMEM_COLS / 64;   // slots at UP = 16
constexpr int AFULL_COUNT = 48;             // items per slot (4, 8, 12, 16) all divide it

// The stage mbarriers and the parity each slot's next phase will have
// (bit s; every barrier completes exactly once per round that uses it).
struct TcBars {
    uint64_t *afull;    // [MAX_SLOTS] A of the slot stored (count AFULL_COUNT)
    uint64_t *dfull;    // [MAX_SLOTS] MMAs of the slot done (one commit)
    uint32_t par;       // phase parity of slot s in bit s (the same for both barriers)
};

template <int UP, bool EXACT>
__device__ __forceinline__ bool stage_tc(float *T, const float *Cs, const PStage &S, int A, int Bv, int NV,
                                         int warp, int lane, uint32_t tmem, TcBars &bars, uint64_t *cbar,
                                         uint32_t cpar) {
    bool coef_ready = false;
    constexpr int NCH = UP / 16;                  // 16-column chunks per slot
    constexpr int SLOTS = TMEM_COLS / (4 * UP);
    constexpr int IPW = (SLOTS * NCH + 3) / 4;    // items per warp in a round (at most)
    const int q = warp & 3, wu = warp >> 2;
    const int MB = S.mb, per = (MB == 64) ? 2 : 1;
    const int ninst = S.G * S.nvb;
    const int ipr = SLOTS * per;                  // instances per round
    const int step = S.sig * A;
    const uint32_t lane_q = static_cast<uint32_t>(32 * q) << 16;
    const int h = (MB == 64) ? (lane >> 4) : 0;
    const int vlane = (MB == 128) ? 32 * q + lane : 16 * q + (lane & 15);

    // tile address of this lane's vector of instance `inst` (element j at + j*step)
    auto lane_base = [&](int inst, bool &ok) -> int {
        const int g = static_cast<int>(fdiv(static_cast<unsigned>(inst), S.f_nvb));
        const int vb = inst - g * S.nvb;
        const int v = vb * MB + vlane;
        ok = inst < ninst && v < NV;
        const int gg = ok ? g : 0, vv = ok ? v : 0;
        const int hi = static_cast<int>(fdiv(static_cast<unsigned>(gg), S.f_sig));
        const int base = hi * (S.b * S.sig) + (gg - hi * S.sig);
        return base * A + vv * Bv;
    };

    for (int i0 = 0; i0 < ninst; i0 += ipr) {
        const int nsl = min(SLOTS, (ninst - i0 + per - 1) / per);
        const int nit = nsl * NCH;                // items per quarter this round
        tc::fence_after_sync();                   // the previous round's TMEM reads are done
        // ---- 1+2. A: split and store this warp's items; the warp of
        // quarter 0 that writes a slot's first chunk then waits for the
        // slot's other items and issues its MMAs right away, so the tensor
        // cores start on early slots while later ones are still written
        bool good = true;
        constexpr uint32_t id1 = tc::idesc_tf32(128, 2 * UP), id2 = tc::idesc_tf32(128, UP);
        constexpr uint32_t id1h = tc::idesc_tf32(64, 2 * UP), id2h = tc::idesc_tf32(64, UP);
#pragma unroll
        for (int u = 0; u < IPW; ++u) {
            const int it = wu + 4 * u;
            if (it >= nit) continue;
            const int sl = it / NCH, c = it - sl * NCH;
            {
                bool ok;
                const int p = lane_base(i0 + sl * per + h, ok);
                const float *xp = T + p + 16 * c * step;
                // every load is unconditional (inputs past b re-read input
                // b-1, lanes without a vector read the tile's first group) and
                // selected afterwards, so the 16 loads issue back to back
                float xv[16], hv[16], lv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int j = EXACT ? i : min(16 * c + i, S.b - 1) - 16 * c;
                    xv[i] = xp[j * step];
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const bool in = EXACT ? ok : (ok && 16 * c + i < S.b);
                    tc::split_tf32(in ? xv[i] : 0.0f, hv[i], lv[i]);
                }
                const uint32_t ta = tmem + lane_q + static_cast<uint32_t>(sl * 4 * UP + 16 * c);
                tc::st16(ta, hv);
                tc::st16(ta + UP, lv);
            }
            tc::wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars.afull[sl], AFULL_COUNT / (4 * NCH));
            if (q == 0 && c == 0) {
                if (!coef_ready) {
                    // this tile's operand blocks of the stage
                    coef_ready = tc::mbar_wait_bounded(cbar, cpar, MMA_WAIT_LIMIT);
                    good = good && coef_ready;
                }
                const bool ready = tc::mbar_wait_bounded(&bars.afull[sl], (bars.par >> sl) & 1u, MMA_WAIT_LIMIT);
                good = good && ready;
                tc::fence_after_sync();
                if (tc::elect_one()) {
                    if (ready && coef_ready) {
                        const uint32_t cbase = tc::smem_u32(Cs) + static_cast<uint32_t>(S.ucoff);
                        for (int hh = 0; hh < per; ++hh) {
                            const int inst = i0 + sl * per + hh;
                            if (inst >= ninst) continue;
                            const int g = static_cast<int>(fdiv(static_cast<unsigned>(inst), S.f_nvb));
                            const uint32_t a = tmem + (static_cast<uint32_t>(16 * hh) << 16) +
                                               static_cast<uint32_t>(sl * 4 * UP);
                            const uint32_t d = a + 2 * UP;
                            const uint32_t bsm = cbase + static_cast<uint32_t>(g * 8 * UP * UP);
#pragma unroll
                            for (int st = 0; st < UP / 8; ++st) {
                                const uint64_t bd =
                                    tc::smem_desc(bsm + static_cast<uint32_t>(st * 64 * UP), 32 * UP, 128);
                                tc::mma_tf32_ts(d, a + 8 * st, bd, MB == 128 ? id1 : id1h, st > 0);
                                tc::mma_tf32_ts(d, a + UP + 8 * st, bd, MB == 128 ? id2 : id2h, 1u);
                            }
                        }
                    }
                    tc::mma_commit(&bars.dfull[sl]);
                }
                __syncwarp();
            }
        }
        // ---- 3. D: for each item of this warp, wait for its slot, load both
        // halves of D, y back into the tile
#pragma unroll
        for (int u = 0; u < IPW; ++u) {
            const int it = wu + 4 * u;
            if (it >= nit) continue;
            const int sl = it / NCH, c = it - sl * NCH;
            good = tc::mbar_wait_bounded(&bars.dfull[sl], (bars.par >> sl) & 1u, MMA_WAIT_LIMIT) && good;
            tc::fence_after_sync();
            const uint32_t td = tmem + lane_q + static_cast<uint32_t>(sl * 4 * UP + 2 * UP + 16 * c);
            float da[16], db[16];
            tc::ld16(td, da);
            tc::ld16(td + UP, db);
            tc::wait_ld();
            if (!good) continue;
            bool ok;
            const int p = lane_base(i0 + sl * per + h, ok);
            float *yp = T + p + 16 * c * step;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const bool out = EXACT ? ok : (ok && 16 * c + i < S.b);
                if (out) yp[i * step] = da[i] + db[i];
            }
        }
        bars.par ^= (1u << nsl) - 1u;             // slots 0..nsl-1 completed one phase each
        tc::fence_before_sync();
        if (__syncthreads_or(good ? 0 : 1)) return false;   // slots free, tile complete
    }
    return true;
}

__device__ __forceinline__ bool stage_tc_any(float *T, const float *Cs, const PStage &S, int A, int Bv, int NV,
                                             int warp, int lane, uint32_t tmem, TcBars &bars, uint64_t *cbar,
                                             uint32_t cpar) {
    const bool ex = (S.b == S.up);
    switch (S.up) {
        case 16: return ex ? stage_tc<16, true>(T, Cs, S, A, Bv, NV, warp, lane, tmem, bars, cbar, cpar)
                           : stage_tc<16, false>(T, Cs, S, A, Bv, NV, warp, lane, tmem, bars, cbar, cpar);
        case 32: return stage_tc<32, false>(T, Cs, S, A, Bv, NV, warp, lane, tmem, bars, cbar, cpar);
        case 48: return stage_tc<48, false>(T, Cs, S, A, Bv, NV, warp, lane, tmem, bars, cbar, cpar);
        default: return stage_tc<64, false>(T, Cs, S, A, Bv, NV, warp, lane, tmem, bars, cbar, cpar);
    }
}

// ------------------------------------------------------------ prologue / epilogue


// Per-tile index tables in shared memory (built once per tile): global row
// offset (row * ld) and global column of every tile row / column, and the
// sign factor of each when the pass applies the sign vectors.
struct Tabs {
    const int64_t *rin, *rout;    // per tile row: input / output offset of its first element
    const int *rtab, *ctab;       // global row / column of each tile row / column
    const int *cin, *cout;        // per tile column: input / output offset
    const float *rsg, *csg;
};

// Scale, code and pack every (row, group) of the tile (last forward pass).
template <int BITS, bool F32COPY>
__device__ __forceinline__ void quantize_tile(const float *T, const PassDesc &D, const QuantDev &Q,
                                              const Tabs &tb, int warp, int lane) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E, TCp = D.TCp;
    const int g = Q.group, ngt = Ec / g, per = g >> 5;
    const bool is_max = Q.stat_max != 0;            // group statistic: max |x| or sum of squares
    const bool lm = (Q.kind == HARP_LLOYD_MAX);
    float t[(1 << BITS) - 1];
#pragma unroll
    for (int k = 0; k < (1 << BITS) - 1; ++k) t[k] = Q.thr[k];
    const int64_t spr = D.cols / g;
    const int64_t wpr = D.cols * BITS / 32;
    const int c0t = tb.ctab[0];
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
        const int64_t row = tb.rtab[tr];
        const int64_t c0 = c0t + gq * g;
        if (lane == 0) D.scales[row * spr + c0 / g] = hb;
        uint32_t *wrow = cw + row * wpr + (c0 / 32) * BITS;
        float *frow = F32COPY ? D.out_f32 + row * D.cols + c0 : nullptr;
        for (int e = 0; e < per; ++e) {
            const float x = rp[lane + 32 * e];
            const int code = code_of<BITS>(x, s, inv, lm, t);
            const unsigned word = pack_words<BITS>(code, lane);
            if (lane < BITS) wrow[e * BITS + lane] = word;
            if constexpr (F32COPY) frow[32 * e + lane] = x;
        }
    }
}

// Tile <-> global moves in units of 4 rows x 32 columns per warp: lane
// (q = lane / 8, c = lane % 8) moves 4 consecutive columns (16 contiguous
// bytes of fp32, 8 of bf16: runs of tile columns are multiples of 4 and
// aligned) of row 4u + q. With an odd pitch the 32 lanes of each shared
// access hit 32 different banks.
struct Quad {
    int tr, tc;
    bool ok;
};

__device__ __forceinline__ Quad quad_of(int u, const FDiv &fnch, int Er, int Ec, int lane) {
    const int rq = static_cast<int>(fdiv(static_cast<unsigned>(u), fnch)), ch = u - rq * static_cast<int>(fnch.d);
    Quad qd;
    qd.tr = 4 * rq + (lane >> 3);
    qd.tc = 32 * ch + 4 * (lane & 7);
    qd.ok = qd.tr < Er && qd.tc < Ec;
    return qd;
}

// Shared tile -> global (fp32 or bf16), times the sign factors when asked.
// A quad goes out as one 16-byte (8-byte) store when its four outputs are
// consecutive and aligned in the output layout, else element by element.
template <int EPI>
__device__ __forceinline__ void store_tile(const float *T, const PassDesc &D, const Tabs &tb, bool signs,
                                           int warp, int lane) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E, TCp = D.TCp;
    const int nch = (Ec + 31) >> 5, nu = ((Er + 3) >> 2) * nch;
    for (int u = warp; u < nu; u += PW) {
        const Quad qd = quad_of(u, D.f_nch, Er, Ec, lane);
        if (!qd.ok) continue;
        const float *t = T + qd.tr * TCp + qd.tc;
        float4 x = make_float4(t[0], t[1], t[2], t[3]);
        if (signs) {
            const float rs = tb.rsg[qd.tr];
            x.x *= rs * tb.csg[qd.tc];
            x.y *= rs * tb.csg[qd.tc + 1];
            x.z *= rs * tb.csg[qd.tc + 2];
            x.w *= rs * tb.csg[qd.tc + 3];
        }
        const int c0 = tb.cout[qd.tc];
        const int64_t off = tb.rout[qd.tr] + c0;
        const bool vec = (tb.cout[qd.tc + 3] == c0 + 3) && ((off & 3) == 0);
        if constexpr (EPI == EPI_BF16) {
            unsigned short *o = static_cast<unsigned short *>(D.out);
            const unsigned short b0 = __bfloat16_as_ushort(__float2bfloat16_rn(x.x));
            const unsigned short b1 = __bfloat16_as_ushort(__float2bfloat16_rn(x.y));
            const unsigned short b2 = __bfloat16_as_ushort(__float2bfloat16_rn(x.z));
            const unsigned short b3 = __bfloat16_as_ushort(__float2bfloat16_rn(x.w));
            if (vec) {
                *reinterpret_cast<uint2 *>(o + off) =
                    make_uint2(b0 | (static_cast<unsigned>(b1) << 16), b2 | (static_cast<unsigned>(b3) << 16));
            } else {
                const int64_t r = tb.rout[qd.tr];
                o[r + c0] = b0;
                o[r + tb.cout[qd.tc + 1]] = b1;
                o[r + tb.cout[qd.tc + 2]] = b2;
                o[r + tb.cout[qd.tc + 3]] = b3;
            }
        } else {
            float *o = static_cast<float *>(D.out);
            if (vec) {
                *reinterpret_cast<float4 *>(o + off) = x;
            } else {
                const int64_t r = tb.rout[qd.tr];
                o[r + c0] = x.x;
                o[r + tb.cout[qd.tc + 1]] = x.y;
                o[r + tb.cout[qd.tc + 2]] = x.z;
                o[r + tb.cout[qd.tc + 3]] = x.w;
            }
        }
    }
}

// Quantiser for 2- and 4-bit codes with groups of a multiple of 32: lane
// (q = lane / 4, c = lane % 4) codes 8 consecutive values of row 8u + q, so
// its 8 codes fill one 32-bit word (4 bits) or half of one (2 bits, joined
// with the neighbouring lane's half). The group statistic adds each lane's
// values in column order, then combines the lanes of the row with a fixed
// xor tree.
template <int BITS, bool F32COPY>
__device__ __forceinline__ void quantize_tile_fast(const float *T, const PassDesc &D, const QuantDev &Q,
                                                   const Tabs &tb, const float *ts, const unsigned char *bins,
                                                   int warp, int lane) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E, TCp = D.TCp;
    const int g = Q.group, ngt = Ec / g, nit = g >> 5;
    const bool is_max = Q.stat_max != 0;            // group statistic: max |x| or sum of squares
    const bool lm = (Q.kind == HARP_LLOYD_MAX);
    const int64_t spr = D.cols / g;
    const int64_t wpr = D.cols * BITS / 32;
    const int q = lane >> 2, c = lane & 3;
    const int nro = (Er + 7) >> 3;
    uint32_t *cw = reinterpret_cast<uint32_t *>(D.codes);
    for (int u = warp; u < nro * ngt; u += PW) {
        const int ro = u / ngt, gq = u - ro * ngt;
        const int tr = 8 * ro + q;
        const bool ok = tr < Er;
        const float *rp = T + min(tr, Er - 1) * TCp + gq * g + 8 * c;
        float st = 0.0f;
        for (int it = 0; it < nit; ++it) {
#pragma unroll
            for (int e = 0; e < 8; ++e) st = combine(st, rp[32 * it + e], is_max);
        }
        float o = __shfl_xor_sync(FULL, st, 1);
        st = is_max ? fmaxf(st, o) : st + o;
        o = __shfl_xor_sync(FULL, st, 2);
        st = is_max ? fmaxf(st, o) : st + o;
        const unsigned short hb = group_scale_bits(st, Q);
        const float s = __half2float(__ushort_as_half(hb));
        const float inv = (s > 0.0f) ? __frcp_rn(s) : 0.0f;
        const int64_t row = tb.rtab[min(tr, Er - 1)];
        const int64_t c0 = tb.ctab[0] + gq * g;
        if (ok && c == 0) D.scales[row * spr + c0 / g] = hb;
        for (int it = 0; it < nit; ++it) {
            unsigned word = 0;
            float x[8];
            if (D.bins && s > 0.0f) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x[e] = rp[32 * it + e];
                    word |= static_cast<unsigned>(code_binned<64>(x[e] * inv, ts, bins)) << (BITS * e);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x[e] = rp[32 * it + e];
                    word |= static_cast<unsigned>(code_of_smem<BITS>(x[e], s, inv, lm, ts)) << (BITS * e);
                }
            }
            const int64_t col = c0 + 32 * it + 8 * c;       // first of this lane's 8 columns
            if constexpr (BITS == 4) {
                if (ok) cw[row * wpr + col / 8] = word;
            } else {
                const unsigned hi = __shfl_down_sync(FULL, word, 1);
                if (ok && (c & 1) == 0) cw[row * wpr + col / 16] = word | (hi << 16);
            }
            if constexpr (F32COPY) {
                if (ok) {
                    float4 *f = reinterpret_cast<float4 *>(D.out_f32 + row * D.cols + col);
                    f[0] = make_float4(x[0], x[1], x[2], x[3]);
                    f[1] = make_float4(x[4], x[5], x[6], x[7]);
                }
            }
        }
    }
}

// ------------------------------------------------------------ the kernel

// One of the two tile buffers in shared memory: tile, coefficient slots,
// and the tile's index tables.
struct Buf {
    float *T, *C;
    Tabs tb;
    int64_t *rin, *rout;
    int *rtab, *ctab, *cin, *cout;
    float *rsg, *csg, *ssc;
};

__device__ __forceinline__ Buf buf_of(float *sm, const PassDesc &D, int b) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E;
    Buf B;
    float *base = sm + D.tile_floats + b * D.buf_floats;
    B.T = sm;
    B.C = D.coef_single ? sm + D.coef_base : base;
    B.rin = reinterpret_cast<int64_t *>(base + D.tab_base);
    B.rout = B.rin + Er;
    B.rtab = reinterpret_cast<int *>(B.rout + Er);
    B.ctab = B.rtab + Er;
    B.cin = B.ctab + Ec;
    B.cout = B.cin + Ec;
    B.rsg = reinterpret_cast<float *>(B.cout + Ec);
    B.csg = B.rsg + Er;
    B.ssc = B.csg + Ec;
    B.tb = Tabs{B.rin, B.rout, B.rtab, B.ctab, B.cin, B.cout, B.rsg, B.csg};
    return B;
}

// Index tables of tile t: global rows / columns, input and output offsets
// (natural row-major with leading dimension ld, or a workspace in tile-major
// order: this pass's for the input, the next pass's for the output), signs.
__device__ __forceinline__ void build_tables(const PassDesc &D, const Buf &B, const int *rloc, const int *cloc,
                                             unsigned t, int64_t ld, int tid) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E;
    const unsigned ntc = static_cast<unsigned>(D.ax[1].nt);
    const unsigned pr = t / ntc, pc = t - pr * ntc;
    const int rb = axis_base(D.ax[0], pr), cb = axis_base(D.ax[1], pc);
    const int64_t E = static_cast<int64_t>(Er) * Ec;
    const int nEc = D.nx[1].E;
    const int64_t nE = static_cast<int64_t>(D.nx[0].E) * nEc;
    const unsigned nntc = static_cast<unsigned>(D.nx[1].nt);
    for (int i = tid; i < Er; i += PT) {
        const int r = rb + rloc[i];
        B.rtab[i] = r;
        B.rin[i] = D.in_blocked ? static_cast<int64_t>(t) * E + static_cast<int64_t>(i) * Ec
                                : static_cast<int64_t>(r) * ld;
        if (D.out_blocked) {
            unsigned p;
            int l;
            axis_local(D.nx[0], r, p, l);
            B.rout[i] = static_cast<int64_t>(p) * nntc * nE + static_cast<int64_t>(l) * nEc;
        } else {
            B.rout[i] = static_cast<int64_t>(r) * ld;
        }
        B.rsg[i] = D.ax[0].sign ? __ldg(D.ax[0].sign + r) : 1.0f;
    }
    for (int i = tid; i < Ec; i += PT) {
        const int c = cb + cloc[i];
        B.ctab[i] = c;
        B.cin[i] = D.in_blocked ? i : c;
        if (D.out_blocked) {
            unsigned p;
            int l;
            axis_local(D.nx[1], c, p, l);
            B.cout[i] = static_cast<int>(p * nE + l);
        } else {
            B.cout[i] = c;
        }
        B.csg[i] = D.ax[1].sign ? __ldg(D.ax[1].sign + c) : 1.0f;
    }
}

// Block coefficients of every stage of a tile into a coefficient buffer
// (asynchronous 16-byte copies; the tile's tables must be built).
__device__ __forceinline__ void issue_coefs(const PassDesc &D, const Tabs &tb, float *C, int warp, int lane) {
    for (int u = 0; u < D.nst; ++u) {
        const PStage &S = D.st[u];
        if (S.had) continue;
        const int cpg = S.jpad * S.kp / 4;
        const int *tab = S.axis == 0 ? tb.rtab : tb.ctab;
        for (int gi = warp; gi < S.G; gi += PW) {
            const int c = global_group(S, tab, gi);
            const float *src = S.coef + static_cast<int64_t>(c) * (S.jpad * S.kp);
            float *dst = C + S.coff + gi * S.gstride;
            for (int o = lane; o < cpg; o += 32) cp_async16(dst + 4 * o, src + 4 * o);
        }
    }
}

// Tensor-core operand blocks of stage u of a tile into the (single)
// coefficient area, by one warp: each of the tile's groups gets its global
// group's 2*up x up block (contiguous in global and shared memory) by one
// bulk copy; `bar` completes when all have landed.
__device__ __forceinline__ void issue_coefs_bulk(const PassDesc &D, const Tabs &tb, float *C, int u, uint64_t *bar,
                                                 int lane) {
    const PStage &S = D.st[u];
    if (S.had) return;
    const int fpg = 2 * S.up * S.up;
    if (lane == 0) tc::mbar_arrive_expect_tx(bar, static_cast<uint32_t>(S.G * fpg * 4));
    __syncwarp();
    const int *tab = S.axis == 0 ? tb.rtab : tb.ctab;
    float *area = C + S.ucoff / 4;
    for (int gi = lane; gi < S.G; gi += 32) {
        const int c = global_group(S, tab, gi);
        tc::bulk_g2s(area + gi * fpg, S.ucoef + static_cast<int64_t>(c) * fpg, static_cast<uint32_t>(fpg * 4), bar);
    }
}

// The next tile's input by bulk copies (one warp), completing on `bar`: the
// whole tile when the input is a workspace in this pass's tile-major order,
// else one copy per tile row (rows of contiguous bf16 values or packed codes).
template <int PRO>
__device__ __forceinline__ void issue_input_bulk(const PassDesc &D, const QuantDev &Q, const Tabs &tb, void *S,
                                                 unsigned t, uint64_t *bar, int lane) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E;
    if (D.in_bulk == 1) {
        const uint32_t bytes = static_cast<uint32_t>(Er * Ec * 4);
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(bar, bytes);
            tc::bulk_g2s(S, static_cast<const float *>(D.in) + static_cast<int64_t>(t) * Er * Ec, bytes, bar);
        }
        return;
    }
    const int rb = D.in_row_bytes;
    if (lane == 0) tc::mbar_arrive_expect_tx(bar, static_cast<uint32_t>(Er * rb));
    __syncwarp();
    for (int tr = lane; tr < Er; tr += 32) {
        const char *src;
        if constexpr (PRO == PRO_CODES)
            src = reinterpret_cast<const char *>(D.in_codes) + static_cast<int64_t>(tb.rtab[tr]) * (D.cols * Q.bits / 8) +
                  static_cast<int64_t>(tb.ctab[0]) * Q.bits / 8;
        else
            src = static_cast<const char *>(D.in) + (tb.rin[tr] + tb.cin[0]) * 2;
        tc::bulk_g2s(static_cast<char *>(S) + tr * rb, src, static_cast<uint32_t>(rb), bar);
    }
}

// Scales of the next codes tile (one register per thread), as issue_input
// loads them.
__device__ __forceinline__ float load_tile_scales(const PassDesc &D, const QuantDev &Q, const Tabs &tb, int tid) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E, ngt = Ec / Q.group;
    float sc = 0.0f;
    if (tid < Er * ngt) {
        const int tr = static_cast<int>(fdiv(static_cast<unsigned>(tid), D.f_ngt)), q = tid - tr * ngt;
        sc = __half2float(__ushort_as_half(__ldg(D.in_scales + static_cast<int64_t>(tb.rtab[tr]) * (D.cols / Q.group) +
                                                 tb.ctab[0] / Q.group + q)));
    }
    return sc;
}

constexpr int MAXCH = 8;   // 32-code chunks per row of a quantised tile (Ec <= 256)


// The next tile's input is copied asynchronously into a dense staging
// buffer (row-major [Er][Ec] fp32 or bf16, or the tile rows' packed code
// words) while the current tile is computed; its scales (codes input) travel
// in one register per thread.
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem));
}

__device__ __forceinline__ void cp_async8(void *smem, const void *gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(s), "l"(gmem));
}

template <int PRO>
__device__ __forceinline__ float issue_input(const PassDesc &D, const QuantDev &Q, const Tabs &tb, void *S, int tid) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E;
    float sc = 0.0f;
    if constexpr (PRO == PRO_CODES) {
        const int wpr = (Ec >> 5) * Q.bits, ngt = Ec / Q.group;
        const int64_t rw = D.cols * Q.bits / 32;
        const uint32_t *words = reinterpret_cast<const uint32_t *>(D.in_codes);
        const int c0 = tb.ctab[0];
        for (int i = tid; i < Er * wpr; i += PT) {
            const int tr = static_cast<int>(fdiv(static_cast<unsigned>(i), D.f_wpr)), w = i - tr * wpr;
            cp_async4(static_cast<uint32_t *>(S) + tr * wpr + w,
                      words + static_cast<int64_t>(tb.rtab[tr]) * rw + (c0 >> 5) * Q.bits + w);
        }
        if (tid < Er * ngt) {
            const int tr = static_cast<int>(fdiv(static_cast<unsigned>(tid), D.f_ngt)), q = tid - tr * ngt;
            sc = __half2float(__ushort_as_half(
                __ldg(D.in_scales + static_cast<int64_t>(tb.rtab[tr]) * (D.cols / Q.group) + c0 / Q.group + q)));
        }
    } else {
        const int nq = Er * (Ec >> 2);                  // quads of 4 consecutive tile columns
        const int nqr = Ec >> 2;
        for (int i = tid; i < nq; i += PT) {
            const int tr = static_cast<int>(fdiv(static_cast<unsigned>(i), D.f_nq)), tc = 4 * (i - tr * nqr);
            const int64_t off = tb.rin[tr] + tb.cin[tc];
            if constexpr (PRO == PRO_F32)
                cp_async16(static_cast<float *>(S) + tr * Ec + tc, static_cast<const float *>(D.in) + off);
            else
                cp_async8(static_cast<unsigned short *>(S) + tr * Ec + tc,
                          static_cast<const unsigned short *>(D.in) + off);
        }
    }
    return sc;
}

// Staging buffer -> fp32 tile (forward sign factors when asked; codes are
// decoded with their group scales).
template <int BITS>
__device__ __forceinline__ void decode_staged(const PassDesc &D, const QuantDev &Q, const uint32_t *S, float *T,
                                              const float *ssc, const float *lev, int warp, int lane) {
    constexpr unsigned MASK = (1u << BITS) - 1u;
    const int Er = D.ax[0].E, Ec = D.ax[1].E, TCp = D.TCp;
    const int nch = Ec >> 5, wpr = nch * BITS, ngt = Ec / Q.group;
    const int bit = lane * BITS, wi = bit >> 5, sh = bit & 31;
    if ((nch & 3) == 0) {
        // a warp unit is one row's 4 consecutive 32-column chunks: each lane
        // decodes column `lane` of each (consecutive lanes store consecutive
        // columns), with the row's index arithmetic paid once per 4 codes
        const int nu4 = nch >> 2;
        for (int u = warp; u < Er * nu4; u += PW) {
            const int tr = static_cast<int>(fdiv(static_cast<unsigned>(u), D.f_nchc4)), ch0 = 4 * (u - tr * nu4);
            const uint32_t *wsrc = S + tr * wpr + ch0 * BITS;
            const float *srow = ssc + tr * ngt;
            float *trow = T + tr * TCp + ch0 * 32 + lane;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                unsigned code = wsrc[k * BITS + wi] >> sh;
                if (sh + BITS > 32) code |= wsrc[k * BITS + wi + 1] << (32 - sh);
                trow[32 * k] = srow[fdiv(static_cast<unsigned>(ch0 + k), D.f_gch)] * lev[code & MASK];
            }
        }
        return;
    }
    for (int u = warp; u < Er * nch; u += PW) {
        const int tr = static_cast<int>(fdiv(static_cast<unsigned>(u), D.f_nchc)), ch = u - tr * nch;
        const uint32_t *wsrc = S + tr * wpr + ch * BITS;
        unsigned code = wsrc[wi] >> sh;
        if (sh + BITS > 32) code |= wsrc[wi + 1] << (32 - sh);
        T[tr * TCp + ch * 32 + lane] =
            ssc[tr * ngt + static_cast<int>(fdiv(static_cast<unsigned>(ch), D.f_gch))] * lev[code & MASK];
    }
}

template <int PRO>
__device__ __forceinline__ void convert_input(const PassDesc &D, const QuantDev &Q, const Tabs &tb, const void *S,
                                              float *T, const float *ssc, const float *lev, bool signs, int tid,
                                              int warp, int lane) {
    const int Er = D.ax[0].E, Ec = D.ax[1].E, TCp = D.TCp;
    if constexpr (PRO == PRO_CODES) {
        const uint32_t *W = static_cast<const uint32_t *>(S);
        if (Q.bits == 2) decode_staged<2>(D, Q, W, T, ssc, lev, warp, lane);
        else if (Q.bits == 3) decode_staged<3>(D, Q, W, T, ssc, lev, warp, lane);
        else decode_staged<4>(D, Q, W, T, ssc, lev, warp, lane);
    } else {
        const int nch = (Ec + 31) >> 5, nu = ((Er + 3) >> 2) * nch;
        for (int u = warp; u < nu; u += PW) {
            const Quad qd = quad_of(u, D.f_nch, Er, Ec, lane);
            if (!qd.ok) continue;
            float4 x;
            if constexpr (PRO == PRO_F32) {
                x = *reinterpret_cast<const float4 *>(static_cast<const float *>(S) + qd.tr * Ec + qd.tc);
            } else {
                const uint2 t = *reinterpret_cast<const uint2 *>(static_cast<const unsigned short *>(S) +
                                                                 qd.tr * Ec + qd.tc);
                x = make_float4(__uint_as_float(t.x << 16), __uint_as_float(t.x & 0xffff0000u),
                                __uint_as_float(t.y << 16), __uint_as_float(t.y & 0xffff0000u));
            }
            if (signs) {
                const float rs = tb.rsg[qd.tr];
                x.x *= rs * tb.csg[qd.tc];
                x.y *= rs * tb.csg[qd.tc + 1];
                x.z *= rs * tb.csg[qd.tc + 2];
                x.w *= rs * tb.csg[qd.tc + 3];
            }
            float *t = T + qd.tr * TCp + qd.tc;
            t[0] = x.x;
            t[1] = x.y;
            t[2] = x.z;
            t[3] = x.w;
        }
    }
}

// Persistent: each CTA walks the tiles blockIdx.x, + gridDim.x, ... The
// next tile's input is loaded into registers and its coefficients copied
// (asynchronously) into the other coefficient buffer before the current
// tile's stages run, so memory latency overlaps the arithmetic.
// Stage paths a build carries: every pass kernel is built three times, so a
// pass runs the build with only the stage code it needs (unused paths cost
// the others registers and instruction-cache room).
enum StageSet {
    SS_ALL = 0,    // Walsh-Hadamard butterflies and all block widths
    SS_BLOCKS = 1, // block stages of any width, no butterfly
    SS_K16 = 2,    // only block stages of exactly 16 outputs and inputs
    SS_TC = 3      // block stages on the tensor cores (3xTF32), Walsh-Hadamard butterflies
};

template <int PRO, int EPI, int SS>
__global__ void __launch_bounds__(PT, 1)
pass_kernel(const __grid_constant__ PassDesc D, const __grid_constant__ QuantDev Q) {
    extern __shared__ float4 sm4[];
    float *sm = reinterpret_cast<float *>(sm4);
    float *T = sm;
    float *lev = sm + D.lev_base;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Er = D.ax[0].E, Ec = D.ax[1].E, TCp = D.TCp;
    const bool has_sign = D.ax[0].sign || D.ax[1].sign;
    const bool load_signs = has_sign && !D.sign_at_store;
    const int64_t ld = (PRO == PRO_CODES) ? D.ld_out : D.ld_in;   // same matrix either side
    const unsigned ntiles = static_cast<unsigned>(D.ax[0].nt * D.ax[1].nt);
    unsigned t = blockIdx.x;
    if (t >= ntiles) return;
    constexpr bool TC = (SS == SS_TC);
    uint32_t tmem = 0;
    TcBars bars{nullptr, nullptr, 0u};
    uint64_t *cbar = nullptr, *ibar = nullptr;
    if constexpr (TC) {
        // the whole TMEM of the SM (one CTA per SM), the per-slot mbarriers
        // of the tensor-core stages, one mbarrier per stage for its operand
        // blocks and one for the next tile's input (bulk copies)
        uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + D.tc_base);
        bars.afull = reinterpret_cast<uint64_t *>(sm + D.tc_base + 2);
        bars.dfull = bars.afull + MAX_SLOTS;
        cbar = bars.dfull + MAX_SLOTS;
        ibar = cbar + MAXPS;
        if (warp == 0) tc::tmem_alloc(tslot, TMEM_COLS);
        if (tid < MAX_SLOTS) {
            tc::mbar_init(&bars.afull[tid], AFULL_COUNT);
            tc::mbar_init(&bars.dfull[tid], 1);
        }
        if (tid < MAXPS) tc::mbar_init(&cbar[tid], 1);
        if (tid == 0) tc::mbar_init(ibar, 1);
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        tmem = *tslot;
    }
    if constexpr (EPI == EPI_QUANT || EPI == EPI_QUANT_F32) {
        // a quantising pass decodes nothing: the level slots hold the bin table
        const int K = 1 << Q.bits;
        if (tid < 16) lev[16 + tid] = (tid < K - 1) ? Q.thr[tid] : __int_as_float(0x7f800000);
        if (D.bins && tid < 64) reinterpret_cast<unsigned char *>(lev)[tid] = bin_entry<64>(tid, Q.thr, K);
    } else if (tid < 16) {
        lev[tid] = Q.level[tid];
        lev[16 + tid] = Q.thr[tid];     // midpoints (Lloyd-Max code search)
    }
    int *rloc = reinterpret_cast<int *>(sm + D.loc_base);   // tile-local part of each global index
    int *cloc = rloc + Er;
    for (int i = tid; i < Er; i += PT) rloc[i] = axis_global(D.ax[0], 0u, i);
    for (int i = tid; i < Ec; i += PT) cloc[i] = axis_global(D.ax[1], 0u, i);
    __syncthreads();

    void *S = sm + D.stage_base;                        // staging buffer of the next tile's input
    float sc_next;
    {
        const Buf B0 = buf_of(sm, D, 0);
        build_tables(D, B0, rloc, cloc, t, ld, tid);
        __syncthreads();
        if constexpr (TC) {
            if (D.in_bulk) {
                if (warp == 0) issue_input_bulk<PRO>(D, Q, B0.tb, S, t, ibar, lane);
                sc_next = (PRO == PRO_CODES) ? load_tile_scales(D, Q, B0.tb, tid) : 0.0f;
            } else {
                sc_next = issue_input<PRO>(D, Q, B0.tb, S, tid);
            }
            if (warp == 1)
                for (int u = 0; u < D.nst; ++u) issue_coefs_bulk(D, B0.tb, B0.C, u, &cbar[u], lane);
        } else {
            sc_next = issue_input<PRO>(D, Q, B0.tb, S, tid);
            issue_coefs(D, B0.tb, B0.C, warp, lane);
        }
        cp_async_commit();
        cp_async_wait_all();
        if constexpr (TC) {
            if (D.in_bulk && !tc::mbar_wait_bounded(ibar, 0u, MMA_WAIT_LIMIT) && tid == 0) atomicOr(&g_pass_fault, 2u);
        }
        if (PRO == PRO_CODES && tid < Er * (Ec / Q.group)) B0.ssc[tid] = sc_next;
        __syncthreads();
        convert_input<PRO>(D, Q, B0.tb, S, T, B0.ssc, lev, load_signs, tid, warp, lane);
        __syncthreads();
    }

    bool fault = false, fault_more = false;
    int fault_k = 0, fault_u = 0;
    for (int k = 0; t < ntiles; ++k, t += gridDim.x) {
        const Buf B = buf_of(sm, D, k & 1);
        const unsigned tn = t + gridDim.x;
        const bool more = tn < ntiles;
        const Buf Bn = buf_of(sm, D, (k + 1) & 1);
        if (more) {
            build_tables(D, Bn, rloc, cloc, tn, ld, tid);
            __syncthreads();
            if (TC && D.in_bulk) {
                if (warp == 0) issue_input_bulk<PRO>(D, Q, Bn.tb, S, tn, ibar, lane);
                sc_next = (PRO == PRO_CODES) ? load_tile_scales(D, Q, Bn.tb, tid) : 0.0f;
            } else {
                sc_next = issue_input<PRO>(D, Q, Bn.tb, S, tid);
            }
            if constexpr (!TC) issue_coefs(D, Bn.tb, Bn.C, warp, lane);
            cp_async_commit();
        }

        for (int u = 0; u < D.nst; ++u) {
            const PStage &S = D.st[u];
            const bool rows = (S.axis == 0);
            const int A = rows ? TCp : 1, Bv = rows ? 1 : TCp, NV = rows ? Ec : Er;
            if constexpr (SS == SS_TC) {
                if (S.had) {
                    switch (S.b) {
                        case 2: stage_fwht<2>(T, S, A, Bv, NV, warp, lane); break;
                        case 4: stage_fwht<4>(T, S, A, Bv, NV, warp, lane); break;
                        case 8: stage_fwht<8>(T, S, A, Bv, NV, warp, lane); break;
                        case 16: stage_fwht<16>(T, S, A, Bv, NV, warp, lane); break;
                        default: stage_fwht<32>(T, S, A, Bv, NV, warp, lane); break;
                    }
                } else {
                    // the stage's issuing warps wait for this tile's operand
                    // blocks (bulk copies issued after the previous tile's stage u)
                    if (!stage_tc_any(T, B.C, S, A, Bv, NV, warp, lane, tmem, bars, &cbar[u],
                                      static_cast<uint32_t>(k & 1))) {
                        fault = true;
                        fault_more = more;
                        fault_k = k;
                        fault_u = u;
                        break;
                    }
                    // the blocks are consumed: bring the next tile's (the stage
                    // ended on a CTA barrier, so the next stage needs no other)
                    if (more && warp == 1) issue_coefs_bulk(D, Bn.tb, Bn.C, u, &cbar[u], lane);
                    continue;
                }
            } else if constexpr (SS == SS_K16) {
                stage_run<16, false, true>(T, B.C, S, A, Bv, NV, warp, lane);
            } else {
                if (SS == SS_ALL && S.had) {
                    switch (S.b) {
                        case 2: stage_fwht<2>(T, S, A, Bv, NV, warp, lane); break;
                        case 4: stage_fwht<4>(T, S, A, Bv, NV, warp, lane); break;
                        case 8: stage_fwht<8>(T, S, A, Bv, NV, warp, lane); break;
                        case 16: stage_fwht<16>(T, S, A, Bv, NV, warp, lane); break;
                        default: stage_fwht<32>(T, S, A, Bv, NV, warp, lane); break;
                    }
                } else if (S.kp == 8) stage_run<8, false>(T, B.C, S, A, Bv, NV, warp, lane);
                else if (S.kp == 16 && S.b == 16 && S.jpad == 16)
                    stage_run<16, false, true>(T, B.C, S, A, Bv, NV, warp, lane);
                else if (S.kp == 16) stage_run<16, false>(T, B.C, S, A, Bv, NV, warp, lane);
                else stage_rounds(T, B.C, S, A, Bv, NV, warp, lane);
            }
            __syncthreads();
        }
        if (fault) break;

        if constexpr (EPI == EPI_QUANT || EPI == EPI_QUANT_F32) {
            constexpr bool F = (EPI == EPI_QUANT_F32);
            const unsigned char *bins = reinterpret_cast<const unsigned char *>(lev);
            if (Q.bits == 2) quantize_tile_fast<2, F>(T, D, Q, B.tb, lev + 16, bins, warp, lane);
            else if (Q.bits == 4) quantize_tile_fast<4, F>(T, D, Q, B.tb, lev + 16, bins, warp, lane);
            else quantize_tile<3, F>(T, D, Q, B.tb, warp, lane);
        } else {
            store_tile<EPI>(T, D, B.tb, D.sign_at_store && has_sign, warp, lane);
        }
        __syncthreads();

        if (more) {
            cp_async_wait_all();
            if constexpr (TC) {
                if (D.in_bulk && !tc::mbar_wait_bounded(ibar, static_cast<uint32_t>((k + 1) & 1), MMA_WAIT_LIMIT) &&
                    tid == 0)
                    atomicOr(&g_pass_fault, 2u);
            }
            if (PRO == PRO_CODES && tid < Er * (Ec / Q.group)) Bn.ssc[tid] = sc_next;
            __syncthreads();
            convert_input<PRO>(D, Q, Bn.tb, S, T, Bn.ssc, lev, load_signs, tid, warp, lane);
            // the staging buffer's reads are ordered before the next bulk copy into it
            if constexpr (TC) tc::fence_proxy_async();
            __syncthreads();
        }
    }

    if constexpr (TC) {
        // copies still in flight land before the CTA leaves; an abandoned
        // batch gets one more bounded wait before its TMEM is released
        cp_async_wait_all();
        if (fault) {
            // every slot's MMAs of the abandoned round (each slot was committed)
            if (tid == 0) atomicOr(&g_pass_fault, 1u);
            if (tid < MAX_SLOTS) tc::mbar_wait_bounded(&bars.dfull[tid], (bars.par >> tid) & 1u, MMA_WAIT_LIMIT);
        }
        // bulk copies for the next tile issued before the fault land before the
        // CTA's shared memory is released
        if (fault) {
            const uint32_t cp = static_cast<uint32_t>(fault_k & 1), np = cp ^ 1u;
            // this tile's blocks of the stages not reached yet, and the next
            // tile's input and blocks issued before the fault
            if (tid >= fault_u && tid < D.nst && !D.st[tid].had) tc::mbar_wait_bounded(&cbar[tid], cp, MMA_WAIT_LIMIT);
            if (fault_more) {
                if (tid == 0 && D.in_bulk) tc::mbar_wait_bounded(ibar, np, MMA_WAIT_LIMIT);
                if (tid < fault_u && !D.st[tid].had) tc::mbar_wait_bounded(&cbar[tid], np, MMA_WAIT_LIMIT);
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        if (warp == 0) {
            tc::fence_after_sync();
            tc::tmem_dealloc(tmem, TMEM_COLS);
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
        const int64_t vs = static_cast<int64_t>(lv) * VL * ((NV + lv * VL - 1) / (lv * VL));
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
    int bits;
};

bool stage_is_fwht(const StageDev &s) { return s.had && s.b <= 32; }

int stage_coef_floats(const PlanDev *pl, int i, int j, int E) {
    int f = 0;
    for (int t = i; t < j; ++t) {
        const StageDev &s = pl->st[t];
        if (!stage_is_fwht(s)) f += (E / s.b) * (s.jpad * s.kp + GPAD);
    }
    return f;
}

int tcp_of(int Ec) { return (Ec % 2 == 0) ? Ec + 1 : Ec; }

// Shared-memory bytes of a tile (layout of PassDesc: tile, coefficients,
// tables, code staging).
// Shared memory of a pass kernel, in floats: the tile (odd pitch), then
// two buffers of block coefficients + index tables (one for the tile being
// computed, one for the next), the tile-local index tables, then 16
// dequantised levels.
struct SmemLayout {
    int tile_floats, coef_floats, tab_base, buf_floats, stage_base, loc_base, lev_base, total_floats;
    int coef_single, coef_base, tc_base;
};

// Which implementation the block stages of the pass kernels use (process-
// wide, harp_set_block_stages): automatic, always the tensor-core build, or
// always the FFMA builds.
int g_block_stage_mode = BLOCK_STAGES_AUTO;

// Whether a pass applying L[iL:jL] and R[iR:jR] runs the tensor-core build.
// It must have a block stage that is not a Walsh-Hadamard butterfly; then,
// automatically, only when one of its blocks is wider than 32: measured on
// the B200 (4096x4096, 4096x11008, 8192x28672 workloads), the tcgen05 stages
// beat the FFMA stages on the 43-wide blocks (a pass with them 17 % faster)
// and lose on blocks of 7, 16 and 32 (passes 10-25 % slower), where the
// per-stage round trip through TMEM costs more than the FFMAs it replaces.
bool pass_uses_tc(const PlanInput &in, int iL, int jL, int iR, int jR) {
    if (g_block_stage_mode == BLOCK_STAGES_FFMA) return false;
    bool blocks = false, wide = false;
    for (int t = iL; in.L && t < jL; ++t)
        if (!stage_is_fwht(in.L->st[t])) {
            blocks = true;
            wide = wide || in.L->st[t].b > 32;
        }
    for (int t = iR; t < jR; ++t)
        if (!stage_is_fwht(in.R->st[t])) {
            blocks = true;
            wide = wide || in.R->st[t].b > 32;
        }
    return blocks && (wide || g_block_stage_mode == BLOCK_STAGES_TC);
}

// Tensor-core operand bytes of the stages [i, j) of one side for a tile
// with E coordinates along that side: (E / b) groups of 2*up*up floats.
int stage_ucoef_floats(const PlanDev *pl, int i, int j, int E) {
    int f = 0;
    for (int t = i; t < j; ++t) {
        const StageDev &s = pl->st[t];
        if (!stage_is_fwht(s)) f += (E / s.b) * 2 * s.up * s.up;
    }
    return f;
}

SmemLayout smem_layout(const PlanInput &in, int iL, int jL, int iR, int jR, int Er, int Ec) {
    SmemLayout L;
    L.coef_single = pass_uses_tc(in, iL, jL, iR, jR) ? 1 : 0;
    L.tile_floats = (Er * tcp_of(Ec) + 31) & ~31;
    int tabs = 2 * Er + 2 * Er + Er + 3 * Ec + Er + Ec;   // rin, rout (int64), rtab, ctab, cin, cout, signs
    if (Ec % in.group == 0) tabs += Er * (Ec / in.group);  // scales of a codes tile
    if (L.coef_single) {
        // tensor-core build: both buffers hold index tables only; one
        // coefficient area (128-byte aligned) is refilled stage by stage
        L.coef_floats = (in.L ? stage_ucoef_floats(in.L, iL, jL, Er) : 0) + stage_ucoef_floats(in.R, iR, jR, Ec);
        L.tab_base = 0;
        L.buf_floats = (tabs + 3) & ~3;
        L.coef_base = (L.tile_floats + 2 * L.buf_floats + 31) & ~31;
        L.stage_base = L.coef_base + L.coef_floats;
    } else {
        L.coef_floats = (in.L ? stage_coef_floats(in.L, iL, jL, Er) : 0) + stage_coef_floats(in.R, iR, jR, Ec);
        L.tab_base = (L.coef_floats + 1) & ~1;
        L.buf_floats = (L.tab_base + tabs + 3) & ~3;
        L.coef_base = 0;
        L.stage_base = L.tile_floats + 2 * L.buf_floats;
    }
    L.loc_base = L.stage_base + Er * Ec;                  // staging: fp32 tile (the largest input form)
    L.lev_base = L.loc_base + ((Er + Ec + 3) & ~3);
    L.tc_base = L.lev_base + 32;                          // TMEM address slot, then 8-byte mbarriers
    L.total_floats = L.tc_base + 2 + 2 * (2 * MAX_SLOTS_HOST + MAXPS + 1) + 2;
    return L;
}

// Best tile for a pass applying L[iL:jL] and R[iR:jR]; `last` passes
// quantise (forward) / decode codes (inverse) and need whole groups of
// contiguous columns; `first` passes may read bf16 pairs.
Cand best_tile(const PlanInput &in, int iL, int jL, int iR, int jR, bool first, bool last, int user_run) {
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
            if (run % 4 || Ec % 4) continue;                // 16-byte f32 / 8-byte bf16 quads
            if (first && run < user_run) continue;          // the pass that reads (writes) the user matrix
            if (last && (Ec % in.group || Ec % 32)) continue;
            if (last && Ec > 32 * MAXCH) continue;          // quantised tiles at most 256 columns wide
            if (smem_layout(in, iL, jL, iR, jR, static_cast<int>(Er), static_cast<int>(Ec)).total_floats * 4 >
                SMEM_BUDGET)
                continue;
            if (Er * Ec > TILE_MAX) continue;
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
bool plan_passes_run(const PlanInput &in, int user_run, std::vector<PassSpec> &out) {
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
                    const Cand c = best_tile(in, iL, jL, iR, jR, iL == 0 && iR == 0, last, user_run);
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

// The user matrix is read (forward) and written (inverse) by the first
// forward pass; its rows are read in runs of at least 16 elements when some
// plan allows it (shorter runs waste most of every 32-byte sector).
bool plan_passes(const PlanInput &in, std::vector<PassSpec> &out) {
    if (in.rows * in.cols >= (int64_t(1) << 31)) return false;
    return plan_passes_run(in, 16, out) || plan_passes_run(in, 4, out);
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
    A.f_nlo = make_fdiv(static_cast<unsigned>(A.nlo));
    A.f_PS = make_fdiv(static_cast<unsigned>(A.P * A.S));
    A.f_S = make_fdiv(static_cast<unsigned>(A.S));
    A.f_Hx = make_fdiv(static_cast<unsigned>(A.Hx));
    A.f_Lx = make_fdiv(static_cast<unsigned>(A.Lx));
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
    int ucoef_floats = 0;
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
        S.had = stage_is_fwht(sd) ? 1 : 0;
        if (!S.had) coef_floats += S.G * S.gstride;
        // tensor-core fields (used by the tcgen05 build)
        const int NV = refs[u].axis == 0 ? D.ax[1].E : D.ax[0].E;
        S.up = sd.up;
        S.mb = NV >= 128 ? 128 : 64;
        S.nvb = (NV + S.mb - 1) / S.mb;
        S.nslots = 512 / (4 * sd.up);
        S.ucoef = inverse ? sd.uinv : sd.ufwd;
        S.ucoff = 4 * ucoef_floats;
        S.f_nvb = make_fdiv(static_cast<unsigned>(S.nvb));
        S.f_sig = make_fdiv(static_cast<unsigned>(S.sig));
        if (!S.had) ucoef_floats += S.G * 2 * sd.up * sd.up;
    }
}

template <int PRO, int EPI, int SS>
int launch_pass_t(const PassDesc &D, const QuantDev &Q, cudaStream_t st) {
    static int attr_done[64] = {};
    static int nsm[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(pass_kernel<PRO, EPI, SS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SMEM_BUDGET);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&nsm[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    const int64_t nb = D.ax[0].nt * D.ax[1].nt;
    if (nb <= 0) return 0;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(nb, nsm[dev]));
    // The tensor-core build takes all 512 TMEM columns of its SM: asking for
    // more than half of the SM's shared memory keeps it to one CTA per SM, so
    // no second CTA ever waits on the allocation.
    const int smem = (SS == SS_TC) ? std::max(D.smem_bytes, TC_MIN_SMEM) : D.smem_bytes;
    pass_kernel<PRO, EPI, SS><<<grid, PT, smem, st>>>(D, Q);
    return cudaGetLastError();
}

template <int PRO, int EPI>
int launch_pass(const PassDesc &D, const QuantDev &Q, cudaStream_t st) {
    if (D.coef_single) return launch_pass_t<PRO, EPI, SS_TC>(D, Q, st);
    bool had = false, k16 = true;
    for (int u = 0; u < D.nst; ++u) {
        had = had || D.st[u].had;
        k16 = k16 && !D.st[u].had && D.st[u].b == 16 && D.st[u].kp == 16 && D.st[u].jpad == 16;
    }
    if (had) return launch_pass_t<PRO, EPI, SS_ALL>(D, Q, st);
    if (k16) return launch_pass_t<PRO, EPI, SS_K16>(D, Q, st);
    return launch_pass_t<PRO, EPI, SS_BLOCKS>(D, Q, st);
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
void build_desc(PassDesc &D, const PlanInput &in, const PassSpec &ps, bool inverse) {
    D = PassDesc{};
    fill_axis(D.ax[0], in.L, ps.iL, ps.jL, ps.XL, in.rows);
    fill_axis(D.ax[1], in.R, ps.iR, ps.jR, ps.XR, in.cols);
    int cf = 0;
    fill_stages(D, in, ps, inverse, cf);
    D.TCp = tcp_of(D.ax[1].E);
    const SmemLayout L = smem_layout(in, ps.iL, ps.jL, ps.iR, ps.jR, D.ax[0].E, D.ax[1].E);
    D.tile_floats = L.tile_floats;
    D.coef_base = L.coef_base;
    D.coef_single = L.coef_single;
    D.tc_base = L.tc_base;
    D.coef_floats = cf;
    D.tab_base = L.tab_base;
    D.buf_floats = L.buf_floats;
    D.lev_base = L.lev_base;
    D.loc_base = L.loc_base;
    D.stage_base = L.stage_base;
    D.f_nq = make_fdiv(static_cast<unsigned>(std::max(1, D.ax[1].E / 4)));
    D.f_nchc = make_fdiv(static_cast<unsigned>(std::max(1, D.ax[1].E / 32)));
    D.f_nchc4 = make_fdiv(static_cast<unsigned>(std::max(1, D.ax[1].E / 128)));
    D.f_nch = make_fdiv(static_cast<unsigned>((D.ax[1].E + 31) / 32));
    D.f_wpr = make_fdiv(static_cast<unsigned>(std::max(1, (D.ax[1].E / 32) * in.bits)));
    D.f_ngt = make_fdiv(static_cast<unsigned>(std::max(1, D.ax[1].E / in.group)));
    D.f_gch = make_fdiv(static_cast<unsigned>(std::max(1, in.group / 32)));
    D.smem_bytes = L.total_floats * 4;
    if (in.L && ps.iL == 0 && ps.jL > 0) D.ax[0].sign = in.L->signs;
    if (ps.iR == 0 && ps.jR > 0) D.ax[1].sign = in.R->signs;
    D.sign_at_store = inverse ? 1 : 0;
    D.cols = in.cols;
}

thread_local void *const *t_events = nullptr;
thread_local int t_nev = 0;

void record_event(int k, cudaStream_t st) {
    if (k < t_nev && t_events[k]) cudaEventRecord(static_cast<cudaEvent_t>(t_events[k]), st);
}

}  // namespace

void set_block_stages(int mode) { g_block_stage_mode = mode; }

int pass_fault_status(unsigned *flags) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_pass_fault, sizeof(v));
    if (e == cudaSuccess && v) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_pass_fault, &zero, sizeof(zero));
    }
    *flags = v;
    return e;
}

void set_pass_events(void *const *events, int n) {
    t_events = (n > 0) ? events : nullptr;
    t_nev = (n > 0) ? n : 0;
}

bool pass_plan_ok(const PlanDev &left, const PlanDev &right, int group) {
    PlanInput in{&left, &right, left.d, right.d, group, 4};
    std::vector<PassSpec> ps;
    return plan_passes(in, ps);
}

int pass_count(const PlanDev &left, const PlanDev &right, int group) {
    PlanInput in{&left, &right, left.d, right.d, group, 4};
    std::vector<PassSpec> ps;
    return plan_passes(in, ps) ? static_cast<int>(ps.size()) : 0;
}

int pass_fma(const PlanDev &left, const PlanDev &right, int group, int k) {
    PlanInput in{&left, &right, left.d, right.d, group, 4};
    std::vector<PassSpec> ps;
    if (!plan_passes(in, ps) || k < 0 || k >= static_cast<int>(ps.size())) return -1;
    int f = 0;
    for (int t = ps[k].iL; t < ps[k].jL; ++t) f += left.st[t].b;
    for (int t = ps[k].iR; t < ps[k].jR; ++t) f += right.st[t].b;
    return f;
}

// Workspace buffers of a plan: the passes hand the matrix on through fp32
// workspaces in the next pass's tile-major order, alternating between two
// buffers of rows*cols floats (one when there are only two passes).
namespace {

void link_passes(PassDesc &D, const PlanInput &in, const std::vector<PassSpec> &ps, int k, bool inverse,
                 float *ws, const void *user_in, void *user_out) {
    const int np = static_cast<int>(ps.size());
    const int64_t n = in.rows * in.cols;
    D.ld_in = in.cols;
    D.ld_out = in.cols;
    if (k == 0) {
        D.in = user_in;
        D.in_blocked = 0;
    } else {
        D.in = ws + ((k - 1) % 2) * n;
        D.in_blocked = 1;
    }
    if (k == np - 1) {
        D.out = user_out;
        D.out_blocked = 0;
    } else {
        D.out = ws + (k % 2) * n;
        D.out_blocked = 1;
        PassDesc Dn;
        build_desc(Dn, in, ps[k + 1], inverse);
        D.nx[0] = Dn.ax[0];
        D.nx[1] = Dn.ax[1];
    }
}

// Whether the tensor-core build can fetch each tile's input with bulk
// copies: the whole tile at once from a workspace in this pass's tile-major
// order, or one copy per tile row when the tile's columns are contiguous and
// every row's run starts and ends on a 16-byte boundary.
void set_bulk_input(PassDesc &D, int pro, int bits, const void *src) {
    D.in_bulk = 0;
    D.in_row_bytes = 0;
    if (!D.coef_single) return;
    if (pro == PRO_F32) {
        if (D.in_blocked) D.in_bulk = 1;
        return;
    }
    const int Ec = D.ax[1].E;
    for (int i = 0; i < Ec; ++i)
        if (axis_global(D.ax[1], 0u, i) != axis_global(D.ax[1], 0u, 0) + i) return;
    if (reinterpret_cast<uintptr_t>(src) % 16) return;
    if (pro == PRO_BF16) {
        if ((Ec * 2) % 16 || (D.ld_in * 2) % 16) return;
        D.in_row_bytes = Ec * 2;
    } else {
        if ((Ec * bits) % 128 || (D.cols * bits / 8) % 16) return;
        D.in_row_bytes = Ec * bits / 8;
    }
    D.in_bulk = 2;
}

}  // namespace

int launch_pass_fwd(const PlanDev &left, const PlanDev &right, const QuantDev &q, const void *in_ptr,
                    int in_dtype, uint8_t *codes, uint16_t *scales, float *rotated_out, float *ws,
                    void *stream) {
    PlanInput in{&left, &right, left.d, right.d, q.group, q.bits};
    std::vector<PassSpec> ps;
    if (!plan_passes(in, ps)) return cudaErrorInvalidValue;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int np = static_cast<int>(ps.size());
    record_event(0, st);
    for (int k = 0; k < np; ++k) {
        const bool first = (k == 0), last = (k == np - 1);
        PassDesc D;
        build_desc(D, in, ps[k], false);
        link_passes(D, in, ps, k, false, ws, in_ptr, nullptr);
        int pro = PRO_F32, epi = EPI_F32;
        if (first) pro = (in_dtype == HARP_BF16) ? PRO_BF16 : PRO_F32;
        set_bulk_input(D, pro, q.bits, D.in);
        if (last) {
            epi = rotated_out ? EPI_QUANT_F32 : EPI_QUANT;
            D.bins = bins_exact(q, 64) ? 1 : 0;
            D.codes = codes;
            D.scales = scales;
            D.out_f32 = rotated_out;
        }
        const int e = dispatch(D, q, pro, epi, st);
        if (e) return e;
        record_event(k + 1, st);
    }
    return 0;
}

int launch_pass_inv(const PlanDev &left, const PlanDev &right, const QuantDev &q, const uint8_t *codes,
                    const uint16_t *scales, void *out, int out_dtype, float *ws, void *stream) {
    PlanInput in{&left, &right, left.d, right.d, q.group, q.bits};
    std::vector<PassSpec> ps;
    if (!plan_passes(in, ps)) return cudaErrorInvalidValue;
    std::reverse(ps.begin(), ps.end());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int np = static_cast<int>(ps.size());
    record_event(0, st);
    for (int k = 0; k < np; ++k) {
        const bool first = (k == 0), last = (k == np - 1);
        PassDesc D;
        build_desc(D, in, ps[k], true);
        link_passes(D, in, ps, k, true, ws, nullptr, out);
        int pro = PRO_F32, epi = EPI_F32;
        if (first) {
            pro = PRO_CODES;
            D.in_codes = codes;
            D.in_scales = scales;
        }
        set_bulk_input(D, pro, q.bits, first ? static_cast<const void *>(codes) : D.in);
        if (last) epi = (out_dtype == HARP_BF16) ? EPI_BF16 : EPI_F32;
        const int e = dispatch(D, q, pro, epi, st);
        if (e) return e;
        record_event(k + 1, st);
    }
    return 0;
}

}  // namespace harp
