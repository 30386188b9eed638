// harp_theta.cu -- a stage's blocks from its int8-stored parameters, built on
// the device.
//
// HARP section 2.2 factors every block as B_{t,c} = Q_{t,c}(theta) G_b: a base
// mixer G_b (the normalised Sylvester matrix for b a power of two, else a
// fixed orthogonal matrix the caller supplies) times a learned orthogonal
// factor, the Givens rotation by theta for b = 2 and the Cayley map
// (I - A)^-1 (I + A) of the skew-symmetric A built from theta for b > 2.
// Section 2.4 keeps the parameters in int8; with a per-stage scale the stored
// value q stands for theta = scale * q.
//
// One CTA builds one group's block at a time (grid-stride over the groups)
// in double precision in shared memory and rounds once to float:
//   1. the augmented matrix [I - A | I + A]  (b x 2b),
//   2. Gauss-Jordan elimination without row exchanges, which leaves
//      diag(p) Q in the right half (p the pivots),
//   3. B = Q G, each entry a b-term dot product divided by its row's pivot.
// No row exchange is needed: the symmetric part of I - A is the identity, so
// every Schur complement met during elimination has a symmetric part >= I
// and every pivot is >= 1 (no zero or tiny pivot, no growth).
// The finished block goes to any of seven layouts at once, so a plan's six
// device copies of a stage are refreshed by one launch.
#include <cuda_runtime.h>

#include "harp_internal.h"

namespace harp {
namespace {

constexpr int kThetaThreads = 256;

// Position of (i, j), i < j, in the row-major strict upper triangle of a
// b x b matrix: rows 0..i-1 hold (b-1) + (b-2) + ... + (b-i) entries.
__device__ __forceinline__ int tri_index(int i, int j, int b) {
    return i * b - i * (i + 1) / 2 + (j - i - 1);
}

__global__ void __launch_bounds__(kThetaThreads)
theta_blocks_kernel(int b, int64_t n_groups, const int8_t *__restrict__ theta, double scale,
                    const float *__restrict__ base, ThetaOut o) {
    extern __shared__ double sm[];
    const int w = 2 * b, bb = b * b;
    double *G = sm;            // [b][b] base mixer
    double *M = G + bb;        // [b][2b] augmented matrix
    double *f = M + b * w;     // [b] elimination factors of one step

    const double rs = 1.0 / sqrt(static_cast<double>(b));
    for (int e = threadIdx.x; e < bb; e += blockDim.x) {
        const int k = e / b, j = e - k * b;
        G[e] = base ? static_cast<double>(base[e]) : ((__popc(k & j) & 1) ? -rs : rs);
    }
    const int64_t P = b > 2 ? static_cast<int64_t>(b) * (b - 1) / 2 : (b == 2 ? 1 : 0);

    for (int64_t c = blockIdx.x; c < n_groups; c += gridDim.x) {
        const int8_t *q = theta + c * P;
        __syncthreads();   // G is ready; the previous group's M has been read
        for (int e = threadIdx.x; e < bb; e += blockDim.x) {
            const int i = e / b, j = e - i * b;
            const double id = (i == j) ? 1.0 : 0.0;
            double lhs = id, rhs = id;
            if (b == 2) {
                // Givens: Q = [[cos a, -sin a], [sin a, cos a]] straight into
                // the right half over an identity left half
                const double a = scale * static_cast<double>(q[0]);
                rhs = (i == j) ? cos(a) : (i < j ? -sin(a) : sin(a));
            } else if (b > 2 && i != j) {
                const double a = (i < j) ? scale * static_cast<double>(q[tri_index(i, j, b)])
                                         : -(scale * static_cast<double>(q[tri_index(j, i, b)]));
                lhs = -a;
                rhs = a;
            }
            M[i * w + j] = lhs;
            M[i * w + b + j] = rhs;
        }
        __syncthreads();
        if (b > 2) {
            for (int k = 0; k < b; ++k) {
                if (threadIdx.x < b) {
                    const int i = threadIdx.x;
                    f[i] = (i == k) ? 0.0 : M[i * w + k] / M[k * w + k];
                }
                __syncthreads();
                // only columns right of k change: columns 0..k are not read
                // again apart from each row's own diagonal entry
                const int nc = w - k - 1;
                for (int e = threadIdx.x; e < b * nc; e += blockDim.x) {
                    const int i = e / nc, j = k + 1 + (e - i * nc);
                    if (i != k) M[i * w + j] -= f[i] * M[k * w + j];
                }
                __syncthreads();
            }
        }
        for (int e = threadIdx.x; e < bb; e += blockDim.x) {
            const int k = e / b, j = e - k * b;
            double acc = 0.0;
            for (int l = 0; l < b; ++l) acc = fma(M[k * w + b + l], G[l * b + j], acc);
            const float v = __double2float_rn(acc / M[k * w + k]);
            if (o.plain) o.plain[(c * b + k) * b + j] = v;
            if (o.fwd) o.fwd[(c * b + j) * o.kpad + k] = v;
            if (o.inv) o.inv[(c * b + k) * o.kpad + j] = v;
            if (o.gfwd) o.gfwd[((j * (o.kpad >> 2) + (k >> 2)) * n_groups + c) * 4 + (k & 3)] = v;
            if (o.pfwd) o.pfwd[(c * o.jp + j) * o.kp + k] = v;
            if (o.pinv) o.pinv[(c * o.jp + k) * o.kp + j] = v;
            if (o.ufwd || o.uinv) {
                // tensor-core operands: tf32-rounded coefficient and remainder
                uint32_t hb, lb;
                asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hb) : "f"(v));
                const float hi = __uint_as_float(hb);
                asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lb) : "f"(v - hi));
                const float lo = __uint_as_float(lb);
                const int64_t ub = c * 2 * o.up * o.up;
                if (o.ufwd) {
                    o.ufwd[ub + umma_block_index(k, j, o.up)] = hi;
                    o.ufwd[ub + umma_block_index(o.up + k, j, o.up)] = lo;
                }
                if (o.uinv) {
                    o.uinv[ub + umma_block_index(j, k, o.up)] = hi;
                    o.uinv[ub + umma_block_index(o.up + j, k, o.up)] = lo;
                }
            }
        }
    }
}

}  // namespace

size_t theta_smem_bytes(int b) {
    return (3 * static_cast<size_t>(b) * b + b) * sizeof(double);
}

int launch_theta_blocks(int b, int64_t n_groups, const int8_t *theta, double scale,
                        const float *base, const ThetaOut &o, void *stream) {
    if (n_groups == 0) return cudaSuccess;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const size_t smem = theta_smem_bytes(b);
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(theta_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    const int64_t grid = n_groups < static_cast<int64_t>(sms) * 8 ? n_groups
                                                                  : static_cast<int64_t>(sms) * 8;
    theta_blocks_kernel<<<static_cast<unsigned>(grid), kThetaThreads, smem,
                          static_cast<cudaStream_t>(stream)>>>(b, n_groups, theta, scale, base, o);
    return cudaGetLastError();
}

}  // namespace harp
