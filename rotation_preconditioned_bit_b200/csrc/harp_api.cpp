// harp_api.cpp -- the C ABI of libharp (declared in include/harp.h): argument
// checking, plan and codebook objects, host-side block and codebook
// construction, and the launch sequences of the fused paths.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <new>
#include <vector>

#include "harp.h"
#include "harp_internal.h"

struct harp_plan_s {
    int device;
    int64_t d;
    int m;
    int32_t radix[HARP_MAX_STAGES];
    void *mem;  // one device allocation: signs, then each stage's fwd and inv blocks
    harp::PlanDev dev;
};

struct harp_codebook_s {
    harp::QuantDev q;
    int K;
};

namespace {

constexpr size_t kMaxTileBytes = 232448;

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_status(int err) { return err == 0 ? HARP_OK : HARP_ERR_CUDA; }

// Whether all n_groups blocks equal the normalised Sylvester Hadamard
// matrix exactly, entry (i, j) = (-1)^popcount(i & j) / sqrt(b) in fp32
// (HARP section 2.2: theta = 0 gives back G_b; b a power of two, 2..64).
bool all_sylvester(int b, int64_t n_groups, const float *B) {
    if (b < 2 || (b & (b - 1)) != 0) return false;
    const float v = static_cast<float>(1.0 / std::sqrt(static_cast<double>(b)));
    for (int64_t c = 0; c < n_groups; ++c)
        for (int i = 0; i < b; ++i)
            for (int j = 0; j < b; ++j) {
                const float e = (__builtin_popcount(static_cast<unsigned>(i & j)) & 1) ? -v : v;
                if (B[(c * b + i) * b + j] != e) return false;
            }
    return true;
}

// Padded block shape of the pass kernels (see StageDev).
int pass_jpad(int b) { return (b + 3) & ~3; }
int pass_kp(int b) { return b <= 8 ? 8 : (b + 15) & ~15; }
int umma_up(int b) { return (b + 15) & ~15; }

// tf32 rounding as tcgen05's tf32 operands see it (10 stored mantissa bits):
// round to nearest, ties away from zero, on the 13 dropped bits.
float tf32_rna(float x) {
    uint32_t u;
    std::memcpy(&u, &x, 4);
    if ((u & 0x7f800000u) != 0x7f800000u) u = (u + 0x1000u) & 0xffffe000u;
    float r;
    std::memcpy(&r, &u, 4);
    return r;
}

// ------------------------------------------------------------ block makers
// HARP (gist.science paper 2605.29843) section 2.2: B = Q(theta) G_b.

// Normalised Sylvester Hadamard, entry (-1)^popcount(i & j) / sqrt(b).
void sylvester(int b, std::vector<double> &H) {
    H.assign(static_cast<size_t>(b) * b, 0.0);
    const double sc = 1.0 / std::sqrt(static_cast<double>(b));
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j)
            H[static_cast<size_t>(i) * b + j] = (__builtin_popcount(static_cast<unsigned>(i & j)) & 1) ? -sc : sc;
}

// Q of G = Q R with diag(R) > 0, by Householder reflections.
bool householder_q(int b, const double *G, std::vector<double> &Q) {
    std::vector<double> R(G, G + static_cast<size_t>(b) * b);
    std::vector<double> V(static_cast<size_t>(b) * b, 0.0);  // reflector k in row k
    std::vector<double> beta(b, 0.0);
    for (int k = 0; k < b; ++k) {
        double nrm = 0.0;
        for (int i = k; i < b; ++i) nrm += R[static_cast<size_t>(i) * b + k] * R[static_cast<size_t>(i) * b + k];
        nrm = std::sqrt(nrm);
        if (nrm == 0.0) return false;
        const double x0 = R[static_cast<size_t>(k) * b + k];
        const double alpha = (x0 >= 0.0) ? -nrm : nrm;
        double vn = 0.0;
        for (int i = k; i < b; ++i) {
            double v = R[static_cast<size_t>(i) * b + k] - (i == k ? alpha : 0.0);
            V[static_cast<size_t>(k) * b + i] = v;
            vn += v * v;
        }
        beta[k] = (vn > 0.0) ? 2.0 / vn : 0.0;
        for (int j = k; j < b; ++j) {           // R <- (I - beta v v^T) R
            double dot = 0.0;
            for (int i = k; i < b; ++i) dot += V[static_cast<size_t>(k) * b + i] * R[static_cast<size_t>(i) * b + j];
            dot *= beta[k];
            for (int i = k; i < b; ++i) R[static_cast<size_t>(i) * b + j] -= dot * V[static_cast<size_t>(k) * b + i];
        }
    }
    // Q = H_0 H_1 ... H_{b-1}: apply the reflectors to I in reverse order
    Q.assign(static_cast<size_t>(b) * b, 0.0);
    for (int i = 0; i < b; ++i) Q[static_cast<size_t>(i) * b + i] = 1.0;
    for (int k = b - 1; k >= 0; --k)
        for (int j = 0; j < b; ++j) {
            double dot = 0.0;
            for (int i = k; i < b; ++i) dot += V[static_cast<size_t>(k) * b + i] * Q[static_cast<size_t>(i) * b + j];
            dot *= beta[k];
            for (int i = k; i < b; ++i) Q[static_cast<size_t>(i) * b + j] -= dot * V[static_cast<size_t>(k) * b + i];
        }
    // make diag(R) positive: flip column k of Q where R[k][k] < 0
    for (int k = 0; k < b; ++k)
        if (R[static_cast<size_t>(k) * b + k] < 0.0)
            for (int i = 0; i < b; ++i) Q[static_cast<size_t>(i) * b + k] = -Q[static_cast<size_t>(i) * b + k];
    return true;
}

// Cayley map (I - A)^-1 (I + A) by Gauss-Jordan elimination with pivoting.
bool cayley(int b, const std::vector<double> &A, std::vector<double> &Q) {
    const int w = 2 * b;
    std::vector<double> M(static_cast<size_t>(b) * w);
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) {
            const double id = (i == j) ? 1.0 : 0.0;
            M[static_cast<size_t>(i) * w + j] = id - A[static_cast<size_t>(i) * b + j];
            M[static_cast<size_t>(i) * w + b + j] = id + A[static_cast<size_t>(i) * b + j];
        }
    for (int c = 0; c < b; ++c) {
        int p = c;
        for (int r = c + 1; r < b; ++r)
            if (std::fabs(M[static_cast<size_t>(r) * w + c]) > std::fabs(M[static_cast<size_t>(p) * w + c])) p = r;
        if (M[static_cast<size_t>(p) * w + c] == 0.0) return false;
        if (p != c)
            for (int j = 0; j < w; ++j) std::swap(M[static_cast<size_t>(p) * w + j], M[static_cast<size_t>(c) * w + j]);
        const double inv = 1.0 / M[static_cast<size_t>(c) * w + c];
        for (int j = 0; j < w; ++j) M[static_cast<size_t>(c) * w + j] *= inv;
        for (int r = 0; r < b; ++r) {
            if (r == c) continue;
            const double f = M[static_cast<size_t>(r) * w + c];
            if (f == 0.0) continue;
            for (int j = 0; j < w; ++j) M[static_cast<size_t>(r) * w + j] -= f * M[static_cast<size_t>(c) * w + j];
        }
    }
    Q.assign(static_cast<size_t>(b) * b, 0.0);
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) Q[static_cast<size_t>(i) * b + j] = M[static_cast<size_t>(i) * w + b + j];
    return true;
}

// ------------------------------------------------------------ Lloyd-Max
// PolarQuant (gist.science paper 2603.29078) section 2: MSE-optimal scalar
// codebook for N(0,1). Solved on the positive half (the optimum is odd-
// symmetric and, for even K, has a threshold at 0): each centroid is its
// cell's conditional mean and each inner threshold the midpoint of its two
// centroids; iterate from evenly spaced levels until nothing moves.
double npdf(double z) { return std::exp(-0.5 * z * z) * 0.39894228040143267794; }

// P(a < Z < b) for 0 <= a < b, from the upper tail to keep precision.
double nmass(double a, double b) {
    const double ta = 0.5 * std::erfc(a * 0.70710678118654752440);
    const double tb = std::isinf(b) ? 0.0 : 0.5 * std::erfc(b * 0.70710678118654752440);
    return ta - tb;
}

bool lloyd_max_half(int K, std::vector<double> &pos) {
    const int n = K / 2;
    pos.resize(n);
    for (int k = 0; k < n; ++k) pos[k] = (k + 0.5) * (3.0 / n);
    std::vector<double> t(n + 1);
    for (int it = 0; it < 1000000; ++it) {
        t[0] = 0.0;
        for (int k = 1; k < n; ++k) t[k] = 0.5 * (pos[k - 1] + pos[k]);
        t[n] = std::numeric_limits<double>::infinity();
        double moved = 0.0;
        for (int k = 0; k < n; ++k) {
            const double hi = std::isinf(t[k + 1]) ? 0.0 : npdf(t[k + 1]);
            const double c = (npdf(t[k]) - hi) / nmass(t[k], t[k + 1]);
            moved = std::fmax(moved, std::fabs(c - pos[k]));
            pos[k] = c;
        }
        if (moved <= 1e-15) return true;
    }
    return true;
}

// Argument checks shared by the two theta entry points.
int theta_args_ok(int b, int64_t n_groups, const int8_t *theta, float theta_scale,
                  const float *base) {
    if (b < 1 || b > HARP_MAX_RADIX) return HARP_ERR_UNSUPPORTED;
    if (n_groups < 0 || !std::isfinite(theta_scale)) return HARP_ERR_INVALID_ARG;
    if (b > 1 && n_groups > 0 && !theta) return HARP_ERR_INVALID_ARG;
    if ((b & (b - 1)) != 0 && !base) return HARP_ERR_INVALID_ARG;
    if (base && !aligned(base, sizeof(float))) return HARP_ERR_ALIGNMENT;
    return HARP_OK;
}

}  // namespace

// ================================================================ C ABI

namespace harp {

int plans_on_current_device(harp_plan_t a, harp_plan_t b) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return HARP_ERR_CUDA; }
    if ((a && a->device != dev) || (b && b->device != dev)) return HARP_ERR_INVALID_ARG;
    return HARP_OK;
}

}  // namespace harp

using harp::plans_on_current_device;

extern "C" {

const char *harp_status_string(int status) {
    switch (status) {
        case HARP_OK: return "ok";
        case HARP_ERR_INVALID_ARG: return "invalid argument";
        case HARP_ERR_SHAPE: return "shape mismatch";
        case HARP_ERR_UNSUPPORTED: return "unsupported configuration";
        case HARP_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
        case HARP_ERR_WORKSPACE: return "workspace missing or too small";
        case HARP_ERR_CUDA: return "CUDA error";
        case HARP_ERR_ALLOC: return "allocation failed";
        default: return "unknown status";
    }
}

int harp_version(void) { return 100; }

int harp_stage_blocks(int kind, int b, int64_t n_groups, const double *gauss,
                      const double *base_gauss, double skew_scale, float *out) {
    if (!out || n_groups < 0) return HARP_ERR_INVALID_ARG;
    if (b < 1 || b > HARP_MAX_RADIX) return HARP_ERR_UNSUPPORTED;
    if (kind != HARP_BLOCKS_HADAMARD && kind != HARP_BLOCKS_QR && kind != HARP_BLOCKS_CAYLEY)
        return HARP_ERR_INVALID_ARG;
    if (kind != HARP_BLOCKS_HADAMARD && !gauss && n_groups > 0) return HARP_ERR_INVALID_ARG;
    const bool pow2 = (b & (b - 1)) == 0;
    std::vector<double> G;
    if (kind != HARP_BLOCKS_QR) {
        if (pow2) {
            sylvester(b, G);
        } else {
            if (!base_gauss) return HARP_ERR_INVALID_ARG;
            if (!householder_q(b, base_gauss, G)) return HARP_ERR_SHAPE;
        }
    }
    const size_t bb = static_cast<size_t>(b) * b;
    std::vector<double> Q, A(bb), B(bb);
    for (int64_t c = 0; c < n_groups; ++c) {
        const double *g = gauss ? gauss + c * bb : nullptr;
        if (kind == HARP_BLOCKS_HADAMARD) {
            B = G;
        } else if (kind == HARP_BLOCKS_QR) {
            if (!householder_q(b, g, B)) return HARP_ERR_SHAPE;
        } else {
            if (b == 2) {
                const double a = skew_scale * g[1];
                Q = {std::cos(a), -std::sin(a), std::sin(a), std::cos(a)};
            } else {
                for (int i = 0; i < b; ++i)
                    for (int j = 0; j < b; ++j)
                        A[static_cast<size_t>(i) * b + j] =
                            (i < j) ? skew_scale * g[static_cast<size_t>(i) * b + j]
                          : (i > j) ? -skew_scale * g[static_cast<size_t>(j) * b + i] : 0.0;
                if (!cayley(b, A, Q)) return HARP_ERR_SHAPE;
            }
            for (int i = 0; i < b; ++i)
                for (int j = 0; j < b; ++j) {
                    double acc = 0.0;
                    for (int k = 0; k < b; ++k) acc += Q[static_cast<size_t>(i) * b + k] * G[static_cast<size_t>(k) * b + j];
                    B[static_cast<size_t>(i) * b + j] = acc;
                }
        }
        for (size_t e = 0; e < bb; ++e) out[c * bb + e] = static_cast<float>(B[e]);
    }
    return HARP_OK;
}

int harp_lloyd_max_centroids(int bits, float *out) {
    if (!out) return HARP_ERR_INVALID_ARG;
    if (bits < 2 || bits > 5) return HARP_ERR_UNSUPPORTED;
    const int K = 1 << bits;
    std::vector<double> pos;
    lloyd_max_half(K, pos);
    for (int k = 0; k < K / 2; ++k) {
        out[K / 2 + k] = static_cast<float>(pos[k]);
        out[K / 2 - 1 - k] = static_cast<float>(-pos[k]);
    }
    return HARP_OK;
}

int harp_plan_create(harp_plan_t *out, int64_t d, int m, const int32_t *radix,
                     const float *const *blocks, const float *signs, void *stream) {
    if (!out || !radix || !blocks) return HARP_ERR_INVALID_ARG;
    *out = nullptr;
    if (m < 1 || m > HARP_MAX_STAGES) return HARP_ERR_UNSUPPORTED;
    if (d < 1 || d > std::numeric_limits<int32_t>::max()) return HARP_ERR_SHAPE;
    int64_t prod = 1;
    for (int t = 0; t < m; ++t) {
        if (radix[t] < 1 || radix[t] > HARP_MAX_RADIX) return HARP_ERR_UNSUPPORTED;
        if (!blocks[t]) return HARP_ERR_INVALID_ARG;
        prod *= radix[t];
        if (prod > d) return HARP_ERR_SHAPE;
    }
    if (prod != d) return HARP_ERR_SHAPE;
    if (static_cast<size_t>(d) * 4 > kMaxTileBytes) return HARP_ERR_UNSUPPORTED;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return HARP_ERR_CUDA; }

    // host staging of the device layout
    const size_t sign_floats = (static_cast<size_t>(d) + 3) & ~static_cast<size_t>(3);
    size_t total = sign_floats;
    std::vector<size_t> off(m), poff(m), uoff(m), goff(m);
    for (int t = 0; t < m; ++t) {
        const int kpad = (radix[t] + 3) & ~3;
        off[t] = total;
        total += 2 * static_cast<size_t>(d) * kpad;   // fwd then inv
    }
    for (int t = 0; t < m; ++t) {                       // row-kernel layout
        goff[t] = total;
        total += static_cast<size_t>(d) * ((radix[t] + 3) & ~3);
    }
    for (int t = 0; t < m; ++t) {                       // pass-kernel layout
        const int b = radix[t];
        poff[t] = total;
        total += 2 * static_cast<size_t>(d / b) * pass_jpad(b) * pass_kp(b);
    }
    for (int t = 0; t < m; ++t) {                       // tensor-core operand layout
        const int up = umma_up(radix[t]);
        uoff[t] = total;
        total += 2 * static_cast<size_t>(d / radix[t]) * 2 * up * up;
    }
    std::vector<float> host;
    try { host.assign(total, 0.0f); } catch (...) { return HARP_ERR_ALLOC; }
    for (int64_t i = 0; i < d; ++i) host[i] = signs ? signs[i] : 1.0f;
    for (int t = 0; t < m; ++t) {
        const int b = radix[t], kpad = (b + 3) & ~3;
        const int64_t ng = d / b;
        float *fwd = host.data() + off[t];
        float *inv = fwd + static_cast<size_t>(d) * kpad;
        for (int64_t c = 0; c < ng; ++c) {
            const float *B = blocks[t] + c * b * b;
            for (int k = 0; k < b; ++k)
                for (int j = 0; j < b; ++j) {
                    fwd[(c * b + j) * kpad + k] = B[k * b + j];
                    inv[(c * b + k) * kpad + j] = B[k * b + j];
                }
        }
        float *gf = host.data() + goff[t];
        for (int64_t c = 0; c < ng; ++c) {
            const float *B = blocks[t] + c * b * b;
            for (int k = 0; k < b; ++k)
                for (int j = 0; j < b; ++j)
                    gf[((static_cast<size_t>(j) * (kpad / 4) + k / 4) * ng + c) * 4 + (k & 3)] = B[k * b + j];
        }
        const int jp = pass_jpad(b), kp = pass_kp(b);
        float *pf = host.data() + poff[t];
        float *pi = pf + static_cast<size_t>(ng) * jp * kp;
        for (int64_t c = 0; c < ng; ++c) {
            const float *B = blocks[t] + c * b * b;
            for (int j = 0; j < b; ++j)
                for (int k = 0; k < b; ++k) {
                    pf[(c * jp + j) * kp + k] = B[k * b + j];
                    pi[(c * jp + j) * kp + k] = B[j * b + k];
                }
        }
        const int up = umma_up(b);
        const size_t ublk = static_cast<size_t>(2) * up * up;
        float *uf = host.data() + uoff[t];
        float *ui = uf + static_cast<size_t>(ng) * ublk;
        for (int64_t c = 0; c < ng; ++c) {
            const float *B = blocks[t] + c * b * b;
            for (int k = 0; k < b; ++k)
                for (int j = 0; j < b; ++j) {
                    const float v = B[k * b + j];
                    const float hi = tf32_rna(v), lo = tf32_rna(v - hi);
                    uf[c * ublk + harp::umma_block_index(k, j, up)] = hi;
                    uf[c * ublk + harp::umma_block_index(up + k, j, up)] = lo;
                    ui[c * ublk + harp::umma_block_index(j, k, up)] = hi;
                    ui[c * ublk + harp::umma_block_index(up + j, k, up)] = lo;
                }
        }
    }
    harp_plan_s *p = new (std::nothrow) harp_plan_s();
    if (!p) return HARP_ERR_ALLOC;
    if (cudaMalloc(&p->mem, total * sizeof(float)) != cudaSuccess) {
        cudaGetLastError();
        delete p;
        return HARP_ERR_ALLOC;
    }
    // ordered on the caller's stream, finished before returning (the host
    // staging copy and the caller's arrays may go away afterwards)
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(p->mem, host.data(), total * sizeof(float), cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaStreamSynchronize(cs) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(p->mem);
        delete p;
        return HARP_ERR_CUDA;
    }
    p->device = dev;
    p->d = d;
    p->m = m;
    for (int t = 0; t < HARP_MAX_STAGES; ++t) p->radix[t] = (t < m) ? radix[t] : 0;
    float *base = static_cast<float *>(p->mem);
    p->dev.d = d;
    p->dev.m = m;
    p->dev.signs = base;
    int64_t s = d;
    for (int t = 0; t < m; ++t) {
        const int b = radix[t], kpad = (b + 3) & ~3;
        s /= b;
        p->dev.st[t].b = b;
        p->dev.st[t].kpad = kpad;
        p->dev.st[t].s = s;
        p->dev.st[t].fwd = base + off[t];
        p->dev.st[t].inv = base + off[t] + static_cast<size_t>(d) * kpad;
        p->dev.st[t].gfwd = base + goff[t];
        p->dev.st[t].jpad = pass_jpad(b);
        p->dev.st[t].kp = pass_kp(b);
        p->dev.st[t].pfwd = base + poff[t];
        p->dev.st[t].pinv = base + poff[t] + static_cast<size_t>(d / b) * pass_jpad(b) * pass_kp(b);
        p->dev.st[t].had = all_sylvester(b, d / b, blocks[t]) ? 1 : 0;
        const int up = umma_up(b);
        p->dev.st[t].up = up;
        p->dev.st[t].ufwd = base + uoff[t];
        p->dev.st[t].uinv = base + uoff[t] + static_cast<size_t>(d / b) * 2 * up * up;
    }
    *out = p;
    return HARP_OK;
}

int harp_plan_destroy(harp_plan_t plan) {
    if (!plan) return HARP_OK;
    int st = HARP_OK;
    if (plan->mem && cudaFree(plan->mem) != cudaSuccess) { cudaGetLastError(); st = HARP_ERR_CUDA; }
    delete plan;
    return st;
}

int harp_theta_blocks(int b, int64_t n_groups, const int8_t *theta, float theta_scale,
                      const float *base, float *out, void *stream) {
    int st = theta_args_ok(b, n_groups, theta, theta_scale, base);
    if (st) return st;
    if (n_groups > 0 && !out) return HARP_ERR_INVALID_ARG;
    if (!aligned(out, sizeof(float))) return HARP_ERR_ALIGNMENT;
    harp::ThetaOut o{};
    o.plain = out;
    return cuda_status(harp::launch_theta_blocks(b, n_groups, theta, theta_scale, base, o, stream));
}

int harp_plan_load_theta(harp_plan_t plan, int stage, const int8_t *theta, float theta_scale,
                         const float *base, void *stream) {
    if (!plan || stage < 0 || stage >= plan->m) return HARP_ERR_INVALID_ARG;
    if (int dv = plans_on_current_device(plan)) return dv;   // the plan's memory lives on its own device
    harp::StageDev &sd = plan->dev.st[stage];
    const int b = sd.b;
    const int64_t ng = plan->d / b;
    int st = theta_args_ok(b, ng, theta, theta_scale, base);
    if (st) return st;
    harp::ThetaOut o{};
    o.fwd = const_cast<float *>(sd.fwd);
    o.inv = const_cast<float *>(sd.inv);
    o.kpad = sd.kpad;
    o.gfwd = const_cast<float *>(sd.gfwd);
    o.pfwd = const_cast<float *>(sd.pfwd);
    o.pinv = const_cast<float *>(sd.pinv);
    o.jp = sd.jpad;
    o.kp = sd.kp;
    o.ufwd = const_cast<float *>(sd.ufwd);
    o.uinv = const_cast<float *>(sd.uinv);
    o.up = sd.up;
    st = cuda_status(harp::launch_theta_blocks(b, ng, theta, theta_scale, base, o, stream));
    if (st == HARP_OK) sd.had = 0;
    return st;
}

int harp_plan_info(harp_plan_t plan, int64_t *d, int *m, int32_t *radix) {
    if (!plan) return HARP_ERR_INVALID_ARG;
    if (d) *d = plan->d;
    if (m) *m = plan->m;
    if (radix) std::memcpy(radix, plan->radix, sizeof(plan->radix));
    return HARP_OK;
}

int harp_codebook_create(harp_codebook_t *out, int kind, int bits, int64_t group, int scale_mode,
                         const float *centroids) {
    if (!out) return HARP_ERR_INVALID_ARG;
    *out = nullptr;
    if (kind != HARP_LLOYD_MAX && kind != HARP_ABSMAX) return HARP_ERR_INVALID_ARG;
    if (scale_mode != HARP_SCALE_RMS && scale_mode != HARP_SCALE_ABSMAX) return HARP_ERR_INVALID_ARG;
    if (bits < 2 || bits > 5) return HARP_ERR_UNSUPPORTED;
    if (group <= 0) return HARP_ERR_SHAPE;
    if (group % 32 != 0 || group > std::numeric_limits<int32_t>::max()) return HARP_ERR_UNSUPPORTED;
    harp_codebook_s *cb = new (std::nothrow) harp_codebook_s();
    if (!cb) return HARP_ERR_ALLOC;
    const int K = 1 << bits;
    cb->K = K;
    cb->q.kind = kind;
    cb->q.bits = bits;
    cb->q.group = static_cast<int>(group);
    if (kind == HARP_LLOYD_MAX) {
        float c[32];
        if (centroids) {
            for (int k = 0; k < K; ++k) c[k] = centroids[k];
            for (int k = 0; k + 1 < K; ++k)
                if (!(c[k] < c[k + 1])) { delete cb; return HARP_ERR_INVALID_ARG; }
            if (scale_mode == HARP_SCALE_ABSMAX && !(c[K - 1] > 0.0f)) { delete cb; return HARP_ERR_INVALID_ARG; }
        } else {
            harp_lloyd_max_centroids(bits, c);
        }
        for (int k = 0; k < K; ++k) cb->q.level[k] = c[k];
        for (int k = 0; k + 1 < K; ++k)
            cb->q.thr[k] = static_cast<float>(0.5 * (static_cast<double>(c[k]) + static_cast<double>(c[k + 1])));
        // default: RMS of the group; absmax mode: max |x| onto the largest centroid
        cb->q.stat_max = (scale_mode == HARP_SCALE_ABSMAX) ? 1 : 0;
        cb->q.scale_div = c[K - 1];
    } else {
        for (int k = 0; k < K; ++k) cb->q.level[k] = static_cast<float>(k - K / 2);
        cb->q.stat_max = 1;
        cb->q.scale_div = static_cast<float>((1 << (bits - 1)) - 1);
    }
    *out = cb;
    return HARP_OK;
}

int harp_codebook_destroy(harp_codebook_t cb) {
    delete cb;
    return HARP_OK;
}

int harp_codebook_tables(harp_codebook_t cb, float *centroids, float *thresholds) {
    if (!cb) return HARP_ERR_INVALID_ARG;
    if (centroids) for (int k = 0; k < cb->K; ++k) centroids[k] = cb->q.level[k];
    if (thresholds) for (int k = 0; k + 1 < cb->K; ++k) thresholds[k] = cb->q.thr[k];
    return HARP_OK;
}

int harp_workspace_size(harp_plan_t left, harp_plan_t right, int64_t rows, int64_t cols,
                        size_t *bytes) {
    (void)right;
    if (!bytes || rows < 0 || cols < 0) return HARP_ERR_INVALID_ARG;
    *bytes = left ? static_cast<size_t>(rows) * static_cast<size_t>(cols) * 8 : 0;
    return HARP_OK;
}

static bool valid_dtype(int t) { return t == HARP_F32 || t == HARP_BF16; }

static size_t dtype_size(int t) { return t == HARP_F32 ? 4 : 2; }

int harp_rotate(harp_plan_t plan, int side, int dir, const void *in, int in_dtype, void *out,
                int out_dtype, int64_t rows, int64_t cols, int64_t ld_in, int64_t ld_out,
                void *stream) {
    if (!plan) return HARP_ERR_INVALID_ARG;
    if (int dv = plans_on_current_device(plan)) return dv;
    if (side != HARP_RIGHT && side != HARP_LEFT) return HARP_ERR_INVALID_ARG;
    if (dir != HARP_FWD && dir != HARP_INV) return HARP_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return HARP_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0) return HARP_ERR_SHAPE;
    if ((side == HARP_RIGHT ? cols : rows) != plan->d) return HARP_ERR_SHAPE;
    if (ld_in < cols || ld_out < cols) return HARP_ERR_SHAPE;
    if (rows == 0 || cols == 0) return HARP_OK;
    if (!in || !out) return HARP_ERR_INVALID_ARG;
    if (ld_in % 4 || ld_out % 4 || !aligned(in, 16) || !aligned(out, 16)) return HARP_ERR_ALIGNMENT;
    const char *ib = static_cast<const char *>(in);
    const char *ob = static_cast<const char *>(out);
    const size_t in_bytes = rows ? (static_cast<size_t>(rows - 1) * ld_in + cols) * dtype_size(in_dtype) : 0;
    const size_t out_bytes = rows ? (static_cast<size_t>(rows - 1) * ld_out + cols) * dtype_size(out_dtype) : 0;
    if (ib < ob + out_bytes && ob < ib + in_bytes) return HARP_ERR_INVALID_ARG;
    harp::VecLaunch L{};
    L.side = side;
    L.dir = dir;
    L.pro = (in_dtype == HARP_F32) ? harp::PRO_F32 : harp::PRO_BF16;
    L.epi = (out_dtype == HARP_F32) ? harp::EPI_F32 : harp::EPI_BF16;
    L.nvec = (side == HARP_RIGHT) ? rows : cols;
    L.in = in;
    L.ld_in = ld_in;
    L.out = out;
    L.ld_out = ld_out;
    return cuda_status(harp::launch_vec(plan->dev, nullptr, L, stream));
}

static int check_codec(harp_codebook_t cb, int64_t rows, int64_t cols) {
    if (!cb) return HARP_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0) return HARP_ERR_SHAPE;
    if (cols % cb->q.group) return HARP_ERR_SHAPE;
    return HARP_OK;
}

int harp_quantize(harp_codebook_t cb, const void *in, int in_dtype, int64_t rows, int64_t cols,
                  int64_t ld_in, uint8_t *codes, uint16_t *scales, void *stream) {
    int st = check_codec(cb, rows, cols);
    if (st) return st;
    if (!valid_dtype(in_dtype)) return HARP_ERR_INVALID_ARG;
    if (ld_in < cols) return HARP_ERR_SHAPE;
    if (rows == 0 || cols == 0) return HARP_OK;
    if (!in || !codes || !scales) return HARP_ERR_INVALID_ARG;
    if (ld_in % 4 || !aligned(in, 16) || !aligned(codes, 4) || !aligned(scales, 2)) return HARP_ERR_ALIGNMENT;
    return cuda_status(harp::launch_quantize(cb->q, in, in_dtype, rows, cols, ld_in, codes, scales, stream));
}

int harp_dequantize(harp_codebook_t cb, const uint8_t *codes, const uint16_t *scales, int64_t rows,
                    int64_t cols, void *out, int out_dtype, int64_t ld_out, void *stream) {
    int st = check_codec(cb, rows, cols);
    if (st) return st;
    if (!valid_dtype(out_dtype)) return HARP_ERR_INVALID_ARG;
    if (ld_out < cols) return HARP_ERR_SHAPE;
    if (rows == 0 || cols == 0) return HARP_OK;
    if (!out || !codes || !scales) return HARP_ERR_INVALID_ARG;
    if (ld_out % 4 || !aligned(out, 16) || !aligned(scales, 2)) return HARP_ERR_ALIGNMENT;
    return cuda_status(harp::launch_dequantize(cb->q, codes, scales, rows, cols, out, out_dtype, ld_out, stream));
}

// Whether a two-sided call runs as pass kernels (their quantizer epilogue and
// code decoding handle 2- to 4-bit codes; 5-bit codes take the whole-vector
// kernels).
static bool use_passes(harp_plan_t left, harp_plan_t right, harp_codebook_t cb) {
    return left && cb->q.bits <= 4 && harp::pass_plan_ok(left->dev, right->dev, cb->q.group);
}

static int check_pair(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, int64_t rows,
                      int64_t cols, void *workspace, size_t ws_bytes) {
    if (!right || !cb) return HARP_ERR_INVALID_ARG;
    int st = plans_on_current_device(left, right);
    if (st) return st;
    st = check_codec(cb, rows, cols);
    if (st) return st;
    if (right->d != cols) return HARP_ERR_SHAPE;
    if (left && left->d != rows) return HARP_ERR_SHAPE;
    if (!use_passes(left, right, cb) &&
        harp::vec_tile(right->dev, harp::EPI_QUANT, cb->q.group) == 0)
        return HARP_ERR_UNSUPPORTED;
    if (left) {
        const size_t need = static_cast<size_t>(rows) * static_cast<size_t>(cols) * 8;
        if (need && (!workspace || ws_bytes < need)) return HARP_ERR_WORKSPACE;
        if (workspace && !aligned(workspace, 16)) return HARP_ERR_ALIGNMENT;
    }
    return HARP_OK;
}

int harp_rotate_quantize(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, const void *in,
                         int in_dtype, int64_t rows, int64_t cols, uint8_t *codes,
                         uint16_t *scales, float *rotated_out, void *workspace, size_t ws_bytes,
                         void *stream) {
    int st = check_pair(left, right, cb, rows, cols, workspace, ws_bytes);
    if (st) return st;
    if (!valid_dtype(in_dtype)) return HARP_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return HARP_OK;
    if (!in || !codes || !scales) return HARP_ERR_INVALID_ARG;
    if (!aligned(in, 16) || !aligned(codes, 4) || !aligned(scales, 2) ||
        (rotated_out && !aligned(rotated_out, 16)) || cols % 4)
        return HARP_ERR_ALIGNMENT;
    if (!left && in_dtype == HARP_BF16 && harp::short_ok(right->dev, harp::SHORT_FWD, 0)) {
        harp::ShortLaunch S{};
        S.mode = harp::SHORT_FWD;
        S.nvec = rows;
        S.in = in;
        S.out = rotated_out;
        S.out_dtype = HARP_F32;
        S.codes = codes;
        S.scales = scales;
        return cuda_status(harp::launch_short(right->dev, cb->q, S, stream));
    }
    if (!left && harp::rows_ok(right->dev, cb->q, in_dtype, in))
        return cuda_status(harp::launch_rows(right->dev, cb->q, in, in_dtype, rows, codes, scales, rotated_out,
                                             stream));
    if (use_passes(left, right, cb))
        return cuda_status(harp::launch_pass_fwd(left->dev, right->dev, cb->q, in, in_dtype, codes, scales,
                                                 rotated_out, static_cast<float *>(workspace), stream));
    const int pro_in = (in_dtype == HARP_F32) ? harp::PRO_F32 : harp::PRO_BF16;
    const void *row_in = in;
    int row_pro = pro_in;
    if (left) {
        harp::VecLaunch Lc{};
        Lc.side = HARP_LEFT;
        Lc.dir = HARP_FWD;
        Lc.pro = pro_in;
        Lc.epi = harp::EPI_F32;
        Lc.nvec = cols;
        Lc.in = in;
        Lc.ld_in = cols;
        Lc.out = workspace;
        Lc.ld_out = cols;
        st = cuda_status(harp::launch_vec(left->dev, nullptr, Lc, stream));
        if (st) return st;
        row_in = workspace;
        row_pro = harp::PRO_F32;
    }
    harp::VecLaunch Lr{};
    Lr.side = HARP_RIGHT;
    Lr.dir = HARP_FWD;
    Lr.pro = row_pro;
    Lr.epi = rotated_out ? harp::EPI_QUANT_F32 : harp::EPI_QUANT;
    Lr.nvec = rows;
    Lr.in = row_in;
    Lr.ld_in = cols;
    Lr.out = rotated_out;
    Lr.ld_out = cols;
    Lr.codes = codes;
    Lr.scales = scales;
    return cuda_status(harp::launch_vec(right->dev, &cb->q, Lr, stream));
}

int harp_requantize(harp_plan_t right, harp_codebook_t cb_in, const uint8_t *codes_in,
                    const uint16_t *scales_in, int64_t rows, int64_t cols, int mid_dtype,
                    void *restored_out, harp_codebook_t cb_out, uint8_t *codes_out,
                    uint16_t *scales_out, void *stream) {
    if (!right || !cb_in || !cb_out) return HARP_ERR_INVALID_ARG;
    if (int dv = plans_on_current_device(right)) return dv;
    if (mid_dtype != HARP_F32 && mid_dtype != HARP_BF16 && mid_dtype != HARP_F16) return HARP_ERR_INVALID_ARG;
    int st = check_codec(cb_in, rows, cols);
    if (st == HARP_OK) st = check_codec(cb_out, rows, cols);
    if (st) return st;
    if (right->d != cols) return HARP_ERR_SHAPE;
    if (harp::vec_tile(right->dev, harp::EPI_REQUANT, cb_out->q.group, harp::PRO_CODES) == 0)
        return HARP_ERR_UNSUPPORTED;
    if (rows == 0 || cols == 0) return HARP_OK;
    if (!codes_in || !scales_in || !codes_out || !scales_out) return HARP_ERR_INVALID_ARG;
    if (!aligned(codes_in, 4) || !aligned(scales_in, 2) || !aligned(codes_out, 4) ||
        !aligned(scales_out, 2) || (restored_out && !aligned(restored_out, 16)))
        return HARP_ERR_ALIGNMENT;
    if (harp::short_ok(right->dev, harp::SHORT_REQUANT, cb_in->q.bits)) {
        harp::ShortLaunch S{};
        S.mode = harp::SHORT_REQUANT;
        S.nvec = rows;
        S.in_codes = codes_in;
        S.in_scales = scales_in;
        S.out = restored_out;
        S.out_dtype = mid_dtype;
        S.codes = codes_out;
        S.scales = scales_out;
        S.q2 = cb_out->q;
        S.mid = mid_dtype;
        return cuda_status(harp::launch_short(right->dev, cb_in->q, S, stream));
    }
    harp::VecLaunch L{};
    L.side = HARP_RIGHT;
    L.dir = HARP_INV;
    L.pro = harp::PRO_CODES;
    L.epi = harp::EPI_REQUANT;
    L.nvec = rows;
    L.in_codes = codes_in;
    L.in_scales = scales_in;
    L.out = restored_out;
    L.ld_out = cols;
    L.codes = codes_out;
    L.scales = scales_out;
    L.q2 = cb_out->q;
    L.mid = mid_dtype;
    return cuda_status(harp::launch_vec(right->dev, &cb_in->q, L, stream));
}

int harp_pass_count(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, int *passes) {
    if (!right || !cb || !passes) return HARP_ERR_INVALID_ARG;
    *passes = use_passes(left, right, cb) ? harp::pass_count(left->dev, right->dev, cb->q.group) : 0;
    return HARP_OK;
}

int harp_pass_fma(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, int pass, int *fma) {
    if (!left || !right || !cb || !fma) return HARP_ERR_INVALID_ARG;
    const int f = harp::pass_fma(left->dev, right->dev, cb->q.group, pass);
    if (f < 0) return HARP_ERR_INVALID_ARG;
    *fma = f;
    return HARP_OK;
}

// ------------------------------------------------------------ host-buffer variants

namespace {

size_t align256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

struct HostScratch {
    size_t values, codes, scales, ws, total;   // byte offsets of the parts, total bytes
    size_t value_bytes, code_bytes, scale_bytes, ws_bytes;
};

int host_scratch(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, int64_t rows, int64_t cols,
                 int value_dtype, HostScratch &h) {
    if (!right || !cb || rows < 0 || cols < 0) return HARP_ERR_INVALID_ARG;
    if (value_dtype != HARP_BF16 && value_dtype != HARP_F32) return HARP_ERR_INVALID_ARG;
    size_t ws = 0;
    int st = harp_workspace_size(left, right, rows, cols, &ws);
    if (st) return st;
    const size_t n = static_cast<size_t>(rows) * static_cast<size_t>(cols);
    h.value_bytes = n * (value_dtype == HARP_BF16 ? 2 : 4);
    h.code_bytes = n * static_cast<size_t>(cb->q.bits) / 8;
    h.scale_bytes = (cb->q.group > 0 ? n / static_cast<size_t>(cb->q.group) : 0) * 2;
    h.ws_bytes = ws;
    h.values = 0;
    h.codes = align256(h.value_bytes);
    h.scales = h.codes + align256(h.code_bytes);
    h.ws = h.scales + align256(h.scale_bytes);
    h.total = h.ws + ws;
    return HARP_OK;
}

}  // namespace

int harp_host_scratch_size(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, int64_t rows,
                           int64_t cols, int value_dtype, size_t *bytes) {
    if (!bytes) return HARP_ERR_INVALID_ARG;
    HostScratch h{};
    const int st = host_scratch(left, right, cb, rows, cols, value_dtype, h);
    if (st) return st;
    *bytes = h.total;
    return HARP_OK;
}

int harp_rotate_quantize_host(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, const void *in,
                              int in_dtype, int64_t rows, int64_t cols, uint8_t *codes, uint16_t *scales,
                              void *dev_scratch, size_t scratch_bytes, void *stream) {
    HostScratch h{};
    int st = host_scratch(left, right, cb, rows, cols, in_dtype, h);
    if (st) return st;
    if (rows == 0 || cols == 0) return HARP_OK;
    if (!in || !codes || !scales) return HARP_ERR_INVALID_ARG;
    if (!dev_scratch || scratch_bytes < h.total) return HARP_ERR_WORKSPACE;
    if (!aligned(dev_scratch, 256)) return HARP_ERR_ALIGNMENT;
    if (int dv = plans_on_current_device(left, right)) return dv;   // before anything is copied
    char *base = static_cast<char *>(dev_scratch);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(base + h.values, in, h.value_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess) {
        cudaGetLastError();
        return HARP_ERR_CUDA;
    }
    st = harp_rotate_quantize(left, right, cb, base + h.values, in_dtype, rows, cols,
                              reinterpret_cast<uint8_t *>(base + h.codes), reinterpret_cast<uint16_t *>(base + h.scales),
                              nullptr, h.ws_bytes ? base + h.ws : nullptr, h.ws_bytes, stream);
    if (st) return st;
    if (cudaMemcpyAsync(codes, base + h.codes, h.code_bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
        cudaMemcpyAsync(scales, base + h.scales, h.scale_bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess) {
        cudaGetLastError();
        return HARP_ERR_CUDA;
    }
    return HARP_OK;
}

int harp_dequantize_unrotate_host(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, const uint8_t *codes,
                                  const uint16_t *scales, int64_t rows, int64_t cols, void *out, int out_dtype,
                                  void *dev_scratch, size_t scratch_bytes, void *stream) {
    HostScratch h{};
    int st = host_scratch(left, right, cb, rows, cols, out_dtype, h);
    if (st) return st;
    if (rows == 0 || cols == 0) return HARP_OK;
    if (!out || !codes || !scales) return HARP_ERR_INVALID_ARG;
    if (!dev_scratch || scratch_bytes < h.total) return HARP_ERR_WORKSPACE;
    if (!aligned(dev_scratch, 256)) return HARP_ERR_ALIGNMENT;
    if (int dv = plans_on_current_device(left, right)) return dv;   // before anything is copied
    char *base = static_cast<char *>(dev_scratch);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(base + h.codes, codes, h.code_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(base + h.scales, scales, h.scale_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess) {
        cudaGetLastError();
        return HARP_ERR_CUDA;
    }
    st = harp_dequantize_unrotate(left, right, cb, reinterpret_cast<const uint8_t *>(base + h.codes),
                                  reinterpret_cast<const uint16_t *>(base + h.scales), rows, cols, base + h.values,
                                  out_dtype, h.ws_bytes ? base + h.ws : nullptr, h.ws_bytes, stream);
    if (st) return st;
    if (cudaMemcpyAsync(out, base + h.values, h.value_bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess) {
        cudaGetLastError();
        return HARP_ERR_CUDA;
    }
    return HARP_OK;
}

int harp_set_block_stages(int mode) {
    if (mode < HARP_BLOCK_STAGES_AUTO || mode > HARP_BLOCK_STAGES_FFMA) return HARP_ERR_INVALID_ARG;
    harp::set_block_stages(mode);
    return HARP_OK;
}

int harp_fault_status(unsigned int *flags) {
    if (!flags) return HARP_ERR_INVALID_ARG;
    unsigned a = 0, b = 0;
    int e = harp::pass_fault_status(&a);
    if (e == 0) e = harp::rows_fault_status(&b);
    *flags = a | b;
    return cuda_status(e);
}

int harp_set_pass_events(void *const *events, int n) {
    if (n < 0 || (n > 0 && !events)) return HARP_ERR_INVALID_ARG;
    harp::set_pass_events(events, n);
    return HARP_OK;
}

int harp_dequantize_unrotate(harp_plan_t left, harp_plan_t right, harp_codebook_t cb,
                             const uint8_t *codes, const uint16_t *scales, int64_t rows,
                             int64_t cols, void *out, int out_dtype, void *workspace,
                             size_t ws_bytes, void *stream) {
    int st = check_pair(left, right, cb, rows, cols, workspace, ws_bytes);
    if (st) return st;
    if (!valid_dtype(out_dtype)) return HARP_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return HARP_OK;
    if (!out || !codes || !scales) return HARP_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(scales, 2) || cols % 4) return HARP_ERR_ALIGNMENT;
    if (!left && harp::short_ok(right->dev, harp::SHORT_INV, cb->q.bits)) {
        harp::ShortLaunch S{};
        S.mode = harp::SHORT_INV;
        S.nvec = rows;
        S.in_codes = codes;
        S.in_scales = scales;
        S.out = out;
        S.out_dtype = out_dtype;
        return cuda_status(harp::launch_short(right->dev, cb->q, S, stream));
    }
    if (use_passes(left, right, cb))
        return cuda_status(harp::launch_pass_inv(left->dev, right->dev, cb->q, codes, scales, out, out_dtype,
                                                 static_cast<float *>(workspace), stream));
    harp::VecLaunch Lr{};
    Lr.side = HARP_RIGHT;
    Lr.dir = HARP_INV;
    Lr.pro = harp::PRO_CODES;
    Lr.nvec = rows;
    Lr.in_codes = codes;
    Lr.in_scales = scales;
    Lr.ld_out = cols;
    if (left) {
        Lr.epi = harp::EPI_F32;
        Lr.out = workspace;
    } else {
        Lr.epi = (out_dtype == HARP_F32) ? harp::EPI_F32 : harp::EPI_BF16;
        Lr.out = out;
    }
    st = cuda_status(harp::launch_vec(right->dev, &cb->q, Lr, stream));
    if (st || !left) return st;
    harp::VecLaunch Lc{};
    Lc.side = HARP_LEFT;
    Lc.dir = HARP_INV;
    Lc.pro = harp::PRO_F32;
    Lc.epi = (out_dtype == HARP_F32) ? harp::EPI_F32 : harp::EPI_BF16;
    Lc.nvec = cols;
    Lc.in = workspace;
    Lc.ld_in = cols;
    Lc.out = out;
    Lc.ld_out = cols;
    return cuda_status(harp::launch_vec(left->dev, nullptr, Lc, stream));
}

}  // extern "C"
