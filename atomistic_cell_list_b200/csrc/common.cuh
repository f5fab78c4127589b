// Shared device helpers for libe2f: status plumbing, bf16 loads, the edge
// frame, real Wigner-D blocks and the radial basis.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/e2f.h"

namespace e2f {

constexpr int kMaxL = 4;

__host__ __device__ constexpr int n_sh(int L) { return (L + 1) * (L + 1); }
// offset of block l in the concatenated Wigner-D storage: sum_{l'<l} (2l'+1)^2
__host__ __device__ constexpr int wig_off(int l) { return l * (4 * l * l - 1) / 3; }
__host__ __device__ constexpr int wig_size(int L) { return wig_off(L + 1); }

static_assert(wig_off(1) == 1 && wig_off(2) == 10 && wig_off(5) == 165, "wigner offsets");

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// number of kernels this library has launched (read by e2f_launch_count)
void count_launch(int n = 1);

#define E2F_CUDA_TRY(expr)                                  \
    do {                                                    \
        cudaError_t e2f_err_ = (expr);                      \
        if (e2f_err_ != cudaSuccess) return E2F_ERR_CUDA;   \
    } while (0)

__device__ __forceinline__ float load_feat(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_feat(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
}

// ---------------------------------------------------------------------------
// Edge frame (gist.science Technical Summary 2.1, "SO(3) -> SO(2) change of
// basis"): a rotation R with R r^ = +z, R = R_y(-theta) R_z(-phi) where theta
// and phi are r^'s polar and azimuthal angles (phi = 0 on the z axis). The
// roll about the axis is free: the SO(2) map commutes with it.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void edge_frame(float x, float y, float z, float R[3][3]) {
    float rho = hypotf(x, y);
    float cp = 1.f, sp = 0.f;
    if (rho > 0.f) { cp = x / rho; sp = y / rho; }
    R[0][0] = z * cp; R[0][1] = z * sp; R[0][2] = -rho;
    R[1][0] = -sp;    R[1][1] = cp;     R[1][2] = 0.f;
    R[2][0] = x;      R[2][1] = y;      R[2][2] = z;
}

// ---------------------------------------------------------------------------
// Real Wigner-D blocks D^l(R), Y_l(R v) = D^l(R) Y_l(v), l = 0..L, by the
// recursion of Ivanic & Ruedenberg (J. Phys. Chem. 100, 6342 (1996); erratum
// J. Phys. Chem. A 102, 9099 (1998)): D^1 is R written in the (y, z, x) order
// of the degree-1 harmonics, and D^l follows from D^1 and D^{l-1} through
// the u, v, w coefficients and the P, U, V, W terms of that paper. Indices
// are resolved at compile time. Output: D[wig_off(l) + (m+l)(2l+1) + (n+l)].
// ---------------------------------------------------------------------------
namespace ir {

// square root evaluated by the compiler (Newton's method in double)
constexpr double csqrt_iter(double x, double cur, double prev) {
    return cur == prev ? cur : csqrt_iter(x, 0.5 * (cur + x / cur), cur);
}
constexpr double csqrt(double x) { return x > 0.0 ? csqrt_iter(x, x > 1.0 ? x : 1.0, 0.0) : 0.0; }

// u, v, w of the recursion for degree l, row m, column n (compile time)
template <int l, int m, int n>
struct Coef {
    static constexpr int am = m < 0 ? -m : m;
    static constexpr double den = (n > -l && n < l) ? double((l + n) * (l - n)) : double((2 * l) * (2 * l - 1));
    static constexpr double d0 = (m == 0) ? 1.0 : 0.0;
    static constexpr float u = float(csqrt(double((l + m) * (l - m)) / den));
    static constexpr float v = float(0.5 * csqrt((1.0 + d0) * double((l + am - 1) * (l + am)) / den) * (1.0 - 2.0 * d0));
    static constexpr float w = float(-0.5 * csqrt(double((l - am - 1) * (l - am)) / den) * (1.0 - d0));
};

template <int l>
__device__ __forceinline__ float Pterm(int i, int a, int b, const float* R1, const float* Dp) {
    // R1[(i+1)*3 + (j+1)], Dp = D^{l-1}: [(a+l-1)*(2l-1) + (b+l-1)]
    constexpr int w = 2 * l - 1;
    auto r1 = [&](int ii, int jj) { return R1[(ii + 1) * 3 + (jj + 1)]; };
    auto dp = [&](int aa, int bb) { return Dp[(aa + l - 1) * w + (bb + l - 1)]; };
    if (b == l) return r1(i, 1) * dp(a, l - 1) - r1(i, -1) * dp(a, -l + 1);
    if (b == -l) return r1(i, 1) * dp(a, -l + 1) + r1(i, -1) * dp(a, l - 1);
    return r1(i, 0) * dp(a, b);
}

template <int l, int m, int n>
__device__ __forceinline__ void entry(const float* R1, const float* Dp, float* Dl) {
    using K = Coef<l, m, n>;
    constexpr int am = K::am;
    float acc = 0.f;
    if constexpr (am < l) acc += K::u * Pterm<l>(0, m, n, R1, Dp);
    float V;
    if constexpr (m == 0) {
        V = Pterm<l>(1, 1, n, R1, Dp) + Pterm<l>(-1, -1, n, R1, Dp);
    } else if constexpr (m > 0) {
        V = Pterm<l>(1, m - 1, n, R1, Dp) * (m == 1 ? 1.41421356237309515f : 1.f);
        if constexpr (m != 1) V -= Pterm<l>(-1, -m + 1, n, R1, Dp);
    } else {
        V = Pterm<l>(-1, -m - 1, n, R1, Dp) * (m == -1 ? 1.41421356237309515f : 1.f);
        if constexpr (m != -1) V += Pterm<l>(1, m + 1, n, R1, Dp);
    }
    acc += K::v * V;
    if constexpr (m != 0 && am < l - 1) {
        const float W = (m > 0) ? Pterm<l>(1, m + 1, n, R1, Dp) + Pterm<l>(-1, -m - 1, n, R1, Dp)
                                : Pterm<l>(1, m - 1, n, R1, Dp) - Pterm<l>(-1, -m + 1, n, R1, Dp);
        acc += K::w * W;
    }
    Dl[(m + l) * (2 * l + 1) + (n + l)] = acc;
}

template <int l, int m, int n>
__device__ __forceinline__ void row(const float* R1, const float* Dp, float* Dl) {
    entry<l, m, n>(R1, Dp, Dl);
    if constexpr (n < l) row<l, m, n + 1>(R1, Dp, Dl);
}

template <int l, int m>
__device__ __forceinline__ void rows(const float* R1, const float* Dp, float* Dl) {
    row<l, m, -l>(R1, Dp, Dl);
    if constexpr (m < l) rows<l, m + 1>(R1, Dp, Dl);
}

template <int l>
__device__ __forceinline__ void step(const float* R1, const float* Dp, float* Dl) {
    rows<l, -l>(R1, Dp, Dl);
}

}  // namespace ir

template <int L>
__device__ __forceinline__ void wigner_blocks(const float R[3][3], float* D) {
    D[0] = 1.f;
    if constexpr (L >= 1) {
        // (y, z, x) order: index 0 <-> y (1), 1 <-> z (2), 2 <-> x (0)
        const int p[3] = {1, 2, 0};
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int b = 0; b < 3; ++b) D[1 + a * 3 + b] = R[p[a]][p[b]];
    }
    if constexpr (L >= 2) ir::step<2>(D + 1, D + wig_off(1), D + wig_off(2));
    if constexpr (L >= 3) ir::step<3>(D + 1, D + wig_off(2), D + wig_off(3));
    if constexpr (L >= 4) ir::step<4>(D + 1, D + wig_off(3), D + wig_off(4));
}

// ---------------------------------------------------------------------------
// Geometry and radial basis (readings of the pages' unstated radial gate):
// r = mic(x_j - x_i); rho_k(d) = u(d) exp(-((d - mu_k)/delta)^2) with
// mu_k = k rc/(n_rbf-1), delta = rc/(n_rbf-1), u(d) = (cos(pi d/rc)+1)/2.
// ---------------------------------------------------------------------------
struct Box {
    float3 len;
    float3 inv;
    int periodic;
};

__device__ __forceinline__ float3 edge_vec(const float* pos, int i, int j, const Box& b) {
    float dx = pos[3 * j + 0] - pos[3 * i + 0];
    float dy = pos[3 * j + 1] - pos[3 * i + 1];
    float dz = pos[3 * j + 2] - pos[3 * i + 2];
    if (b.periodic) {
        dx -= b.len.x * rintf(dx * b.inv.x);
        dy -= b.len.y * rintf(dy * b.inv.y);
        dz -= b.len.z * rintf(dz * b.inv.z);
    }
    return make_float3(dx, dy, dz);
}

__device__ __forceinline__ float rbf(float d, int k, float cutoff, int n_rbf) {
    const float step = cutoff / float(n_rbf - 1);
    const float t = (d - float(k) * step) / step;
    const float u = 0.5f * (cosf(3.14159265358979323846f * d / cutoff) + 1.f);
    return u * expf(-t * t);
}

// all n_rbf basis values of one distance (the envelope evaluated once);
// out[k] = 0 for n_rbf <= k < NMAX (unrolled: out stays in registers)
template <int NMAX>
__device__ __forceinline__ void rbf_all(float d, float cutoff, int n_rbf, float* out) {
    const float step = cutoff / float(n_rbf - 1);
    const float u = 0.5f * (cosf(3.14159265358979323846f * d / cutoff) + 1.f);
#pragma unroll
    for (int k = 0; k < NMAX; ++k) {
        const float t = (d - float(k) * step) / step;
        out[k] = k < n_rbf ? u * expf(-t * t) : 0.f;
    }
}

}  // namespace e2f
