// Internal interface between the C ABI (harp_api.cpp) and the kernels
// (harp_kernels.cu). Not installed; the public surface is include/harp.h.
#pragma once

#include <cmath>
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "harp.h"

namespace harp {

// One stride stage as the kernels see it. Blocks are stored twice, padded
// along the output index to a multiple of 4 so a lane reads four outputs'
// coefficients with one 16-byte load:
//   fwd[c][j][k] = B_{t,c}[k][j]   (forward: out k, in j)
//   inv[c][k][j] = B_{t,c}[k][j]   (inverse applies B^T: out j, in k)
// both [d/b][b][kpad] floats, zero in the padding.
struct StageDev {
    int b;
    int kpad;
    int64_t s;
    const float *fwd;
    const float *inv;
    // The same blocks for the pass kernels, [d/b][jpad][kp] floats with
    // jpad = b rounded up to 4 and kp = b rounded up to 8 (b <= 8) or 16:
    //   pfwd[c][j][k] = B_{t,c}[k][j],  pinv[c][j][k] = B_{t,c}[j][k]
    // (coefficient of input j in output k), zero in the padding.
    int jpad;
    int kp;
    const float *pfwd;
    const float *pinv;
    // 1 when every block of the stage is exactly the normalised Sylvester
    // Hadamard matrix (fp32 entries +-1/sqrt(b), b a power of two): the pass
    // kernels then apply the stage as a fast Walsh-Hadamard butterfly.
    int had;
    // The same blocks as tensor-core operands for the pass kernels' 3xTF32
    // stages (split-precision products on tcgen05.mma kind::tf32): up = b
    // rounded up to 16; per group 2*up x up floats, K-major "core matrix"
    // order (8 operand rows x 4 inputs per 128-byte unit):
    //   float index (kk/4)*8*up + (n/8)*32 + (n%8)*4 + kk%4
    // for operand row n (output) and input kk. Rows n < up hold the
    // tf32-rounded coefficients (hi), rows up + n the tf32-rounded remainders
    // (lo = coefficient - hi). ufwd: output k, input j -> B[k][j]; uinv:
    // output j, input k -> B[k][j] (the transposed blocks). Zero in padding.
    int up;
    const float *ufwd;
    const float *uinv;
    // The forward blocks interleaved across the stage's G = d/b groups for
    // the row kernel, whose consecutive threads own consecutive groups:
    //   gfwd[((j * kpad/4 + k/4) * G + c) * 4 + k%4] = B_{t,c}[k][j]
    // (one float4 of four outputs' coefficients of input j per group, so a
    // warp's 16-byte loads are contiguous), zero in the padding.
    const float *gfwd;
};

// Operand float index of (row n, input kk) in a tensor-core block of
// padded size up (see StageDev).
__host__ __device__ inline int umma_block_index(int n, int kk, int up) {
    return (kk >> 2) * 8 * up + (n >> 3) * 32 + (n & 7) * 4 + (kk & 3);
}

struct PlanDev {
    int64_t d;
    int m;
    const float *signs;  // [d] +-1 (always present; all ones when none given)
    StageDev st[HARP_MAX_STAGES];
};

// Quantizer tables travel by value as a kernel argument.
struct QuantDev {
    int kind;       // HARP_LLOYD_MAX | HARP_ABSMAX
    int bits;
    int group;
    int stat_max;   // group statistic: 1 = max |x| (absmax, or Lloyd-Max with HARP_SCALE_ABSMAX), 0 = sum of squares
    float scale_div;  // scale = statistic / scale_div when stat_max (qmax, or the largest centroid)
    float level[32];  // dequantised level per code (centroid or code - 2^(b-1))
    float thr[32];    // Lloyd-Max midpoints (K - 1 used)
};

// Whether the binned Lloyd-Max code search (code_binned<nb>: nb bins of
// width 8/nb over [-4, 4], the edge bins open-ended) is exact for q's fp32
// midpoints, i.e. no bin holds two of them. Absmax codebooks never use it.
inline bool bins_exact(const QuantDev &q, int nb) {
    if (q.kind != HARP_LLOYD_MAX) return false;
    const int K = 1 << q.bits;
    int prev = -1;
    for (int k = 0; k < K - 1; ++k) {
        // bin i covers [(i - nb/2 - 1/2) * 8/nb, (i - nb/2 + 1/2) * 8/nb)
        int bin = static_cast<int>(std::floor(static_cast<double>(q.thr[k]) * (nb / 8.0) + nb / 2.0 + 0.5));
        bin = bin < 0 ? 0 : (bin > nb - 1 ? nb - 1 : bin);
        if (bin == prev) return false;
        prev = bin;
    }
    return true;
}

enum Prologue { PRO_F32 = 0, PRO_BF16 = 1, PRO_CODES = 2 };
enum Epilogue { EPI_F32 = 0, EPI_BF16 = 1, EPI_QUANT = 2, EPI_QUANT_F32 = 3, EPI_REQUANT = 4 };

// Launch parameters of the whole-vector kernel: `nvec` vectors of length
// plan.d taken from a row-major matrix, either its rows (side RIGHT) or its
// columns (side LEFT).
struct VecLaunch {
    int side;
    int dir;
    int pro;
    int epi;
    int64_t nvec;
    const void *in;
    int64_t ld_in;
    void *out;             // EPI_F32 / EPI_BF16 / EPI_QUANT_F32 (fp32 copy)
    int64_t ld_out;
    uint8_t *codes;        // EPI_QUANT*: packed codes, row stride = d*bits/8
    uint16_t *scales;      // EPI_QUANT*: [nvec][d/group]
    const uint8_t *in_codes;     // PRO_CODES
    const uint16_t *in_scales;   // PRO_CODES
    // EPI_REQUANT: the second quantizer (codes / scales above are its
    // outputs) and the restored weights' storage type (HARP_F32 | HARP_BF16 |
    // HARP_F16); `out` (optional) receives the restored weights in that type.
    QuantDev q2;
    int mid;
};

// Returns a cudaError_t value (0 = success).
int launch_vec(const PlanDev &plan, const QuantDev *q, const VecLaunch &L, void *stream);
int launch_quantize(const QuantDev &q, const void *in, int in_dtype, int64_t rows, int64_t cols,
                    int64_t ld_in, uint8_t *codes, uint16_t *scales, void *stream);
int launch_dequantize(const QuantDev &q, const uint8_t *codes, const uint16_t *scales,
                      int64_t rows, int64_t cols, void *out, int out_dtype, int64_t ld_out,
                      void *stream);

// Pass kernels (harp_pass.cu): the two-sided paths as a short sequence of
// tiled passes over the matrix, each applying a run of stages of both
// processors to a digit-box tile held in shared memory. `ws` is an fp32
// rows x cols workspace; every pass updates its tiles in place.
// pass_plan_ok: whether such a plan exists for these processors and group.
bool pass_plan_ok(const PlanDev &left, const PlanDev &right, int group);
int pass_count(const PlanDev &left, const PlanDev &right, int group);
// FMAs per element of forward pass k (sum of its radices), -1 if none.
int pass_fma(const PlanDev &left, const PlanDev &right, int group, int k);
int launch_pass_fwd(const PlanDev &left, const PlanDev &right, const QuantDev &q, const void *in,
                    int in_dtype, uint8_t *codes, uint16_t *scales, float *rotated_out, float *ws,
                    void *stream);
int launch_pass_inv(const PlanDev &left, const PlanDev &right, const QuantDev &q,
                    const uint8_t *codes, const uint16_t *scales, void *out, int out_dtype,
                    float *ws, void *stream);

// Implementation of the pass kernels' block stages (harp_set_block_stages).
enum BlockStages { BLOCK_STAGES_AUTO = 0, BLOCK_STAGES_TC = 1, BLOCK_STAGES_FFMA = 2 };
void set_block_stages(int mode);

// Reads and clears the pass kernels' record of bounded waits that ran out
// on the current device (cudaError_t; synchronous).
int pass_fault_status(unsigned *flags);

// Timing hook of the pass launchers (harp_set_pass_events): when n > 0,
// every fused call records events[0] before its first pass and events[k+1]
// after pass k (k + 1 < n). Per calling thread.
void set_pass_events(void *const *events, int n);

// Stage blocks from int8-stored parameters (harp_theta.cu): B_c = Q(theta_c)
// G_b for n_groups groups, theta = scale * q, written to every non-null
// layout of ThetaOut. Returns a cudaError_t value.
struct ThetaOut {
    float *plain;   // [c][k][j] = B[k][j]
    float *fwd;     // [(c b + j) kpad + k] = B[k][j]
    float *inv;     // [(c b + k) kpad + j] = B[k][j]
    int kpad;
    float *pfwd;    // [(c jp + j) kp + k] = B[k][j]
    float *pinv;    // [(c jp + k) kp + j] = B[k][j]
    int jp;
    int kp;
    float *ufwd;    // tensor-core operand blocks (StageDev::ufwd / uinv), up = padded size
    float *uinv;
    int up;
    float *gfwd;    // group-interleaved forward blocks (StageDev::gfwd), same kpad
};
size_t theta_smem_bytes(int b);
int launch_theta_blocks(int b, int64_t n_groups, const int8_t *theta, double scale,
                        const float *base, const ThetaOut &o, void *stream);

// Short-vector kernel (harp_short.cu): row-side calls with d = 32, 64 or
// 128, one thread per vector. Modes: forward (bf16 rows -> codes + scales,
// optional fp32 rotated copy in `out`), inverse (codes -> rows in
// out_dtype), requantize (codes -> restored rows in `mid` (optionally
// stored in `out`) -> codes + scales of q2).
enum ShortMode { SHORT_FWD = 0, SHORT_INV = 1, SHORT_REQUANT = 2 };
struct ShortLaunch {
    int mode;
    int64_t nvec;
    const void *in;              // SHORT_FWD: bf16 [nvec][d]
    const uint8_t *in_codes;     // SHORT_INV / SHORT_REQUANT
    const uint16_t *in_scales;
    void *out;                   // optional except SHORT_INV
    int out_dtype;               // HARP_F32 | HARP_BF16 | HARP_F16
    uint8_t *codes;              // SHORT_FWD / SHORT_REQUANT outputs
    uint16_t *scales;
    QuantDev q2;                 // SHORT_REQUANT: the second quantizer
    int mid;                     // SHORT_REQUANT: restored storage type
    int bins;                    // set by launch_short: binned Lloyd-Max code search
};
bool short_ok(const PlanDev &P, int mode, int in_bits);
int launch_short(const PlanDev &P, const QuantDev &q, const ShortLaunch &L, void *stream);

// Row kernel (harp_rows.cu): right-only rotate + quantize of whole rows for
// processors with radices 2, 4, 8, 16 and d up to 8192 (contiguous rows).
bool rows_ok(const PlanDev &P, const QuantDev &q, int in_dtype, const void *in);
int launch_rows(const PlanDev &P, const QuantDev &q, const void *in, int in_dtype, int64_t rows, uint8_t *codes,
                uint16_t *scales, float *rotated_out, void *stream);
int rows_fault_status(unsigned *flags);

// A plan's blocks live in device memory of the device that was current when
// it was created; a launch from another device would read them through a
// foreign address. HARP_OK when every non-null plan belongs to the current
// device, HARP_ERR_INVALID_ARG otherwise (HARP_ERR_CUDA without a device).
// Every entry point that launches checks this before anything else.
int plans_on_current_device(harp_plan_t a, harp_plan_t b = nullptr);

// Vectors per CTA the whole-vector kernel uses for this plan and epilogue
// (0 if a vector does not fit in shared memory).
int vec_tile(const PlanDev &plan, int epi, int group, int pro = PRO_F32);

}  // namespace harp
