// Backward of the on-the-fly equivariant attention. fp32 CUDA cores; with
// bf16 storage the SO(2) maps and their transposes run on tensor cores
// (m16n8k16 mma.sync, fp16 operands, fp32 accumulation), and the SO(2)
// weight gradient is a GEMM over edges on operand rows built once per edge
// chunk (cuBLAS, fp16 operands, fp32 accumulation).
//
// The pages' conservative variant takes forces as the negative gradient of
// the energy with respect to the positions (E2Former-V2, gist.science
// Technical Summary 2.2 and the experiments on molecular dynamics), so the
// layer's backward pass follows its forward. Given G = dLoss/dout [N, K, C],
// this file computes dLoss / d(pos, x, W_q, W_k, W_rad, W_so2) in the same
// recompute style as the forward: per-edge quantities (frame, Wigner blocks,
// gates, rotated features, SO(2) outputs) are rebuilt on chip and never
// stored per edge, except for one scalar per edge and head and, with bf16
// storage, the weight gradient's operand rows of one chunk of edges.
//
// Per edge e = (i <- j) with alpha = softmax weight, X~ = D(g_v . x_j),
// Y = F(X~) (the SO(2) maps), v = D^T Y, out_i = sum_e alpha v:
//   beta^h   = sum_{c in h} <D G_i, Y>                 (= <G_i, v> per head)
//   dY       = alpha D G_i,   dX~ = F^T(dY)
//   dx_j    += g_v . D^T dX~,  dg_v = sum_m x_j . D^T dX~
//   dW_so2   = sum_e dY (x) X~   (A and B blocks; a tile kernel, or GEMMs over edges)
//   da^h     = alpha^h (beta^h - delta_i^h),  delta_i^h = sum_e alpha beta
//   logits a = g_a <q_i, k_j>/sqrt(d): dq_i, dk_j, dg_a
//   gates    [g_v | g_a] = rho(d) W_rad: dW_rad, dd through rho'(d)
//   direction: for the rotation exp(eps Omega_a) R (Omega_a = e_a x, a = x, y)
//     dLoss/deps_a = <dD_a (alpha G_i), Y> + <dX~, dD_a (g_v . x_j)>,
//     with dD_a = d/deps D(exp(eps Omega_a) R); the direction moves by
//     R^T e_y (a = x) and -R^T e_x (a = y), so the tangential part of
//     dLoss/dr is (dL/deps_x R^T e_y - dL/deps_y R^T e_x) / d.
//   dpos_j += dLoss/dr,  dpos_i -= dLoss/dr  (r = mic(pos_j - pos_i)).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <cuda.h>
#include <cublas_v2.h>
#include <dlfcn.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <type_traits>

#include "attention.cuh"
#include "common.cuh"
#include "tcgen05.cuh"

#define E2F_CUDA_TRY_E(expr)                          \
    do {                                              \
        const cudaError_t e2f_e_ = (expr);            \
        if (e2f_e_ != cudaSuccess) return e2f_e_;     \
    } while (0)

namespace e2f {
namespace bwd {

constexpr int kNt = 256;     // threads of the weight-gradient kernel
constexpr int kNodeNt = 512; // threads of the node kernel (one CTA per SM: 16 warps hide latency)
constexpr int kTe = 8;       // edges per tile of the node kernel
constexpr int kDwR = 128;    // weight-gradient tile rows
constexpr int kDwC = 64;     // weight-gradient tile columns
constexpr int kDwE = 32;     // edges per operand sub-chunk of the weight-gradient kernel
constexpr int kDwChunk = 128;  // edges per geometry chunk (one per thread)
constexpr int kDwSplit = 8;    // edge ranges per tile (partial sums added in a fixed order)

struct BwdParams {
    int n_atoms, C, H, n_rbf, M;
    int n_pairs;
    float cutoff;
    Box box;
    const float* pos;
    const int32_t* row_ptr;
    const int32_t* col;
    const void* x;
    const void* W;     // packed SO(2) weights as given (row-major blocks)
    const float* Wt;   // the same, fp32, each block transposed
    const float* Wrad;
    const float* q;
    const float* k;
    const float* G;    // dLoss/dout
    float* lse;        // [N, H]
    float* beta;       // [E, H]
    float* gq;         // [N, C]
    float* gk;         // [N, C]
    float* gpos;       // [N, 3]
    float* gx;         // [N, K, C]
    float* gWrad;      // [n_rbf, G]
    float* gW;         // packed like W
    const __half* w16;   // W in fp16, row-major blocks (bf16 storage: tensor-core maps)
    const __half* wt16;  // the same, each block transposed
    float* gWpart;     // [kDwSplit][so2 total] partial sums of gW
    int dw_tiles;      // tiles of the SO(2) blocks
    int* status;       // device status word (bounded waits that ran out)
};

// Derivative of the Wigner blocks along dR (R -> R + eps dR): the recursion
// D^l = step(D^1, D^{l-1}) is bilinear in its two arguments, so
// dD^l = step(dD^1, D^{l-1}) + step(D^1, dD^{l-1}), with dD^1 = dR in the
// (y, z, x) order of the degree-1 harmonics.
template <int L>
__device__ __forceinline__ void wigner_dblocks(const float* D, const float dR[3][3], float* dD) {
    dD[0] = 0.f;
    if constexpr (L >= 1) {
        const int p[3] = {1, 2, 0};
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int b = 0; b < 3; ++b) dD[1 + a * 3 + b] = dR[p[a]][p[b]];
    }
    float t[81];
    if constexpr (L >= 2) {
        ir::step<2>(dD + 1, D + wig_off(1), dD + wig_off(2));
        ir::step<2>(D + 1, dD + wig_off(1), t);
        for (int a = 0; a < 25; ++a) dD[wig_off(2) + a] += t[a];
    }
    if constexpr (L >= 3) {
        ir::step<3>(dD + 1, D + wig_off(2), dD + wig_off(3));
        ir::step<3>(D + 1, dD + wig_off(2), t);
        for (int a = 0; a < 49; ++a) dD[wig_off(3) + a] += t[a];
    }
    if constexpr (L >= 4) {
        ir::step<4>(dD + 1, D + wig_off(3), dD + wig_off(4));
        ir::step<4>(D + 1, dD + wig_off(3), t);
        for (int a = 0; a < 81; ++a) dD[wig_off(4) + a] += t[a];
    }
}

// radial basis value and its derivative in d (the forward's rbf)
__device__ __forceinline__ void rbf_and_deriv(float d, int k, float cutoff, int n_rbf, float& v, float& dv) {
    const float step = cutoff / float(n_rbf - 1);
    const float t = (d - float(k) * step) / step;
    const float ang = 3.14159265358979323846f * d / cutoff;
    const float u = 0.5f * (cosf(ang) + 1.f);
    const float du = -0.5f * (3.14159265358979323846f / cutoff) * sinf(ang);
    const float ex = expf(-t * t);
    v = u * ex;
    dv = du * ex + u * ex * (-2.f * t / step);
}

// logit of edge (i <- j), head h, and the pieces its gradient needs
struct Logit {
    float a, ga, dot;
};
__device__ __forceinline__ Logit edge_logit(const BwdParams& P, int i, int j, int h, int Gv, int G, float inv,
                                            float3* u_out, float* d_out, float* gap_out) {
    const float3 r = edge_vec(P.pos, i, j, P.box);
    const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
    float ga = 0.f, gap = 0.f;
    for (int kb = 0; kb < P.n_rbf; ++kb) {
        float v, dv;
        rbf_and_deriv(d, kb, P.cutoff, P.n_rbf, v, dv);
        const float w = P.Wrad[(size_t)kb * G + Gv + h];
        ga = fmaf(v, w, ga);
        gap = fmaf(dv, w, gap);
    }
    const int dh = P.C / P.H;
    const float* qi = P.q + (size_t)i * P.C + h * dh;
    const float* kj = P.k + (size_t)j * P.C + h * dh;
    float dot = 0.f;
    for (int c = 0; c < dh; ++c) dot = fmaf(qi[c], kj[c], dot);
    if (u_out) *u_out = make_float3(r.x / d, r.y / d, r.z / d);
    if (d_out) *d_out = d;
    if (gap_out) *gap_out = gap;
    return Logit{ga * dot * inv, ga, dot};
}

// m16n8k16 fp16 x fp16 -> fp32 (A row-major 16 x 16, B col-major 16 x 8)
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Wigner blocks in shared memory with every row padded to 12 floats (three
// float4): row `row` (0..2l) of block l starts at 12 (l^2 + row)
constexpr int kPRow = 12;
__host__ __device__ constexpr int wig_padded(int L) { return kPRow * (L + 1) * (L + 1); }
__device__ __forceinline__ void ld_row(const float* p, float* d) {
#pragma unroll
    for (int v = 0; v < kPRow / 4; ++v) *reinterpret_cast<float4*>(d + 4 * v) = reinterpret_cast<const float4*>(p)[v];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// fp16 operand rows of the tensor-core maps: (L+1)C + 8 halves (conflict-free fragment loads)
__host__ __device__ inline int node_np(int L, int C) { return (L + 1) * C + 8; }

size_t node_smem_floats(int L, int C, int H, int n_rbf, bool tc) {
    (void)tc;  // the fp16 operands of the tensor-core maps live in the fp32 X~ region
    const int K = n_sh(L), WS = wig_size(L), Gv = (L + 1) * C, G = Gv + H;
    const int KH = (L >= 1) ? std::max((L + 1) * C, 2 * L * C) : C;
    const int KHS = std::max(KH, node_np(L, C));  // the X~ region also holds the fp16 operands
    (void)WS;
    return (size_t)K * C + 3ull * kTe * wig_padded(L) + 2ull * kTe * n_rbf + (size_t)kTe * G + (size_t)kTe * Gv +
           2ull * kTe * H + 12ull * kTe + (size_t)(KHS + 2 * KH) * kTe + (size_t)n_rbf * G + C + 2ull * H + 4 + kTe +
           2ull * kNodeNt + kTe;
}

// One CTA per destination node at a time (persistent over nodes): every
// gradient except dW_so2, dW_q, dW_k and the l = 0 part of dx that flows
// through q and k.
template <int L, typename T>
__global__ void __launch_bounds__(kNodeNt, 1) k_bwd_node(BwdParams P) {
    constexpr int K = n_sh(L);
    constexpr int WS = wig_size(L);
    const int C = P.C, H = P.H, dh = C / H, nr = P.n_rbf, M = P.M;
    const int Gv = (L + 1) * C, G = Gv + H;
    const int KH = (L >= 1) ? max((L + 1) * C, 2 * L * C) : C;
    const T* __restrict__ x = static_cast<const T*>(P.x);
    const T* __restrict__ W = static_cast<const T*>(P.W);

    extern __shared__ float sm[];
    float* Gi = sm;                    // [K][C] dLoss/dout_i
    constexpr int WP = wig_padded(L);
    float* Dm = Gi + K * C;            // [te][WP] Wigner blocks, rows padded
    float* Dx = Dm + kTe * WP;         // [te][WP] their derivative along Omega_x
    float* Dy = Dx + kTe * WP;         // [te][WP] ... along Omega_y
    float* rho = Dy + kTe * WP;        // [te][nr]
    float* rhop = rho + kTe * nr;      // [te][nr] d rho / d d
    float* g = rhop + kTe * nr;        // [te][G] gates
    float* dgv = g + kTe * G;          // [te][Gv] dLoss/dg_v
    float* alpha = dgv + kTe * Gv;     // [te][H]
    float* beta = alpha + kTe * H;     // [te][H]
    float* geo = beta + kTe * H;       // [te][12]: r^ (3), d, R^T e_y (3), -R^T e_x (3), dL/deps_x, dL/deps_y
    float* hs = geo + 12 * kTe;        // [KH][te] gated rotated input of the |m| block
    float* gy = hs + max(KH, node_np(L, C)) * kTe;  // [KH][te] D G_i, then dLoss/dY = alpha D G_i
    float* yb = gy + KH * kTe;         // [KH][te] Y = F(X~) of the block
    float* gWr = yb + KH * kTe;        // [nr][G] this CTA's part of dW_rad
    float* gqi = gWr + nr * G;         // [C]
    float* lse_s = gqi + C;            // [H]
    float* dlt = lse_s + H;            // [H] delta_i
    float* gpi = dlt + H;              // [4] dpos_i
    float* ddv = gpi + 4;              // [te]
    float* red = ddv + kTe;            // [2 kNodeNt]
    int* jn = reinterpret_cast<int*>(red + 2 * kNodeNt);  // [te]
    // bf16 storage: the SO(2) maps and their transposes run as m16n8k16 tensor-core products
    // with fp16 operands, [s][e][np] in the hs region: X~ until the maps are done, then dY
    constexpr bool TC = std::is_same<T, __nv_bfloat16>::value;
    const int np = node_np(L, C);
    __half* hs16 = reinterpret_cast<__half*>(hs);
    __half* gy16 = hs16;

    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, t4 = lane & 3, nwarp = nt / 32;
    const float inv = rsqrtf((float)dh);
    for (int t = tid; t < nr * G; t += nt) gWr[t] = 0.f;

    for (int i = blockIdx.x; i < P.n_atoms; i += gridDim.x) {
        const int e_begin = P.row_ptr[i], e_end = P.row_ptr[i + 1], deg = e_end - e_begin;
        __syncthreads();
        for (int t = tid; t < K * C; t += nt) Gi[t] = P.G[(size_t)i * K * C + t];
        for (int t = tid; t < C; t += nt) gqi[t] = 0.f;
        if (tid < H) dlt[tid] = 0.f;
        if (tid < 4) gpi[tid] = 0.f;
        // softmax statistics of node i (thread t: head t % H)
        {
            const int h = tid % H;
            float mh = -INFINITY, sh = 0.f;
            for (int e = tid / H; e < deg; e += nt / H) {
                const Logit lg = edge_logit(P, i, P.col[e_begin + e], h, Gv, G, inv, nullptr, nullptr, nullptr);
                const float mn = fmaxf(mh, lg.a);
                sh = sh * expf(mh - mn) + expf(lg.a - mn);
                mh = mn;
            }
            red[tid] = mh;
            red[nt + tid] = sh;
        }
        __syncthreads();
        if (tid < H) {
            float mh = -INFINITY, sh = 0.f;
            for (int t = tid; t < nt; t += H) {
                const float mo = red[t], so = red[nt + t];
                if (mo == -INFINITY) continue;
                const float mn = fmaxf(mh, mo);
                sh = ((mh == -INFINITY) ? 0.f : sh * expf(mh - mn)) + so * expf(mo - mn);
                mh = mn;
            }
            lse_s[tid] = (deg > 0) ? mh + logf(sh) : 0.f;
            P.lse[(size_t)i * H + tid] = lse_s[tid];
        }
        __syncthreads();

        for (int e0 = e_begin; e0 < e_end; e0 += kTe) {
            const int ne = min(kTe, e_end - e0);
            // geometry, frame, Wigner blocks and their two tangential derivatives
            if (tid < kTe) {
                const int e = tid;
                float* gg = geo + e * 12;
                if (e < ne) {
                    const int j = P.col[e0 + e];
                    jn[e] = j;
                    const float3 r = edge_vec(P.pos, i, j, P.box);
                    const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
                    float R[3][3];
                    edge_frame(r.x / d, r.y / d, r.z / d, R);
                    // the recursion writes the blocks unpadded at the start of the edge's slots;
                    // then every entry moves up to its padded place (12 (l^2 + row) + n >=
                    // wig_off(l) + row (2l+1) + n), highest first, and the padding is zeroed
                    float* De = Dm + e * WP;
                    float* Xe = Dx + e * WP;
                    float* Ye = Dy + e * WP;
                    wigner_blocks<L>(R, De);
                    float dR[3][3];
#pragma unroll
                    for (int c = 0; c < 3; ++c) { dR[0][c] = 0.f; dR[1][c] = -R[2][c]; dR[2][c] = R[1][c]; }
                    wigner_dblocks<L>(De, dR, Xe);
#pragma unroll
                    for (int c = 0; c < 3; ++c) { dR[0][c] = R[2][c]; dR[1][c] = 0.f; dR[2][c] = -R[0][c]; }
                    wigner_dblocks<L>(De, dR, Ye);
                    for (int l = L; l >= 0; --l) {
                        const int w = 2 * l + 1;
                        for (int row = w - 1; row >= 0; --row)
                            for (int n = w - 1; n >= 0; --n) {
                                const int o = kPRow * (l * l + row) + n, q = wig_off(l) + row * w + n;
                                De[o] = De[q];
                                Xe[o] = Xe[q];
                                Ye[o] = Ye[q];
                            }
                    }
                    for (int l = 0; l <= L; ++l) {
                        const int w = 2 * l + 1;
                        for (int row = 0; row < w; ++row)
                            for (int n = w; n < kPRow; ++n) {
                                const int o = kPRow * (l * l + row) + n;
                                De[o] = 0.f;
                                Xe[o] = 0.f;
                                Ye[o] = 0.f;
                            }
                    }
                    for (int kb = 0; kb < nr; ++kb) rbf_and_deriv(d, kb, P.cutoff, nr, rho[e * nr + kb], rhop[e * nr + kb]);
                    gg[0] = r.x / d; gg[1] = r.y / d; gg[2] = r.z / d; gg[3] = d;
                    gg[4] = R[1][0]; gg[5] = R[1][1]; gg[6] = R[1][2];
                    gg[7] = -R[0][0]; gg[8] = -R[0][1]; gg[9] = -R[0][2];
                } else {
                    jn[e] = i;
                    for (int a = 0; a < WP; ++a) { Dm[e * WP + a] = 0.f; Dx[e * WP + a] = 0.f; Dy[e * WP + a] = 0.f; }
                    for (int kb = 0; kb < nr; ++kb) { rho[e * nr + kb] = 0.f; rhop[e * nr + kb] = 0.f; }
                    for (int a = 0; a < 10; ++a) gg[a] = 0.f;
                    gg[3] = 1.f;
                }
                gg[10] = 0.f;
                gg[11] = 0.f;
            }
            __syncthreads();
            for (int t = tid; t < kTe * G; t += nt) {
                const int e = t / G, c = t % G;
                float s = 0.f;
                for (int kb = 0; kb < nr; ++kb) s = fmaf(rho[e * nr + kb], P.Wrad[(size_t)kb * G + c], s);
                g[t] = s;
            }
            for (int t = tid; t < kTe * Gv; t += nt) dgv[t] = 0.f;
            __syncthreads();
            for (int t = tid; t < kTe * H; t += nt) {
                const int e = t / H, h = t % H;
                float al = 0.f;
                if (e < ne) {
                    const float* qi = P.q + (size_t)i * C + h * dh;
                    const float* kj = P.k + (size_t)jn[e] * C + h * dh;
                    float dot = 0.f;
                    for (int c = 0; c < dh; ++c) dot = fmaf(qi[c], kj[c], dot);
                    al = expf(g[e * G + Gv + h] * dot * inv - lse_s[h]);
                }
                alpha[t] = al;
                beta[t] = 0.f;
            }
            __syncthreads();

#pragma unroll 1
            for (int m = 0; m <= M; ++m) {
                const int nm = (L + 1 - m) * C;
                // gated rotated input X~ of the block: hs[(s, l1-m, c)][e]
                for (int t = tid; t < kTe * nm; t += nt) {
                    const int e = t / nm, r = t % nm;
                    const int l1 = m + r / C, c = r % C;
                    float vp = 0.f, vm = 0.f;
                    if (e < ne) {
                        const int w = 2 * l1 + 1;
                        const size_t xb = ((size_t)jn[e] * K + l1 * l1) * C + c;
                        float xr[2 * L + 1];  // all loads issued before the arithmetic
#pragma unroll
                        for (int n = 0; n < 2 * L + 1; ++n) xr[n] = (n < w) ? load_feat(x, xb + (size_t)n * C) : 0.f;
                        float dp_[kPRow], dm_[kPRow];
                        ld_row(Dm + e * WP + kPRow * (l1 * l1 + l1 + m), dp_);
                        ld_row(Dm + e * WP + kPRow * (l1 * l1 + l1 - m), dm_);
#pragma unroll
                        for (int n = 0; n < 2 * L + 1; ++n) {
                            vp = fmaf(dp_[n], xr[n], vp);
                            vm = fmaf(dm_[n], xr[n], vm);
                        }
                        const float gv = g[e * G + l1 * C + c];
                        vp *= gv;
                        vm *= gv;
                    }
                    if constexpr (TC) {
                        hs16[(size_t)e * np + r] = __float2half_rn(vp);
                        if (m > 0) hs16[(size_t)(kTe + e) * np + r] = __float2half_rn(vm);
                    } else {
                        hs[(size_t)r * kTe + e] = vp;
                        if (m > 0) hs[(size_t)(nm + r) * kTe + e] = vm;
                    }
                }
                __syncthreads();
                // Y = F(X~) row by row; beta, the first direction term, dY = alpha D G_i
                const float* At = P.Wt + so2_offset(L, C, m, 0);
                const float* Bt = (m > 0) ? P.Wt + so2_offset(L, C, m, 1) : nullptr;
                if constexpr (TC) {
                    // Y+ = A X+ - B X-, Y- = B X+ + A X-: one warp per 16 rows, N = the tile's 8 edges
                    const __half* Aw = P.w16 + so2_offset(L, C, m, 0);
                    const __half* Bw = P.w16 + so2_offset(L, C, m, 1);
                    for (int rb = warp; rb < nm / 16; rb += nwarp) {
                        float yp[4] = {0.f, 0.f, 0.f, 0.f}, ym[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                        for (int k0 = 0; k0 < nm; k0 += 16) {
                            const size_t fo = (((size_t)rb * (nm >> 4) + (k0 >> 4)) * 32 + lane) * 8;
                            uint32_t aa[4];
                            *reinterpret_cast<uint4*>(aa) = *reinterpret_cast<const uint4*>(Aw + fo);
                            const __half* xp = hs16 + (size_t)g8 * np + k0 + 2 * t4;
                            const uint32_t xp0 = *reinterpret_cast<const uint32_t*>(xp);
                            const uint32_t xp1 = *reinterpret_cast<const uint32_t*>(xp + 8);
                            mma16816(yp, aa, xp0, xp1);
                            if (m > 0) {
                                uint32_t ab[4], an[4];
                                *reinterpret_cast<uint4*>(ab) = *reinterpret_cast<const uint4*>(Bw + fo);
#pragma unroll
                                for (int q = 0; q < 4; ++q) an[q] = ab[q] ^ 0x80008000u;
                                const __half* xm = hs16 + (size_t)(kTe + g8) * np + k0 + 2 * t4;
                                const uint32_t xm0 = *reinterpret_cast<const uint32_t*>(xm);
                                const uint32_t xm1 = *reinterpret_cast<const uint32_t*>(xm + 8);
                                mma16816(yp, an, xm0, xm1);
                                mma16816(ym, ab, xp0, xp1);
                                mma16816(ym, aa, xm0, xm1);
                            }
                        }
                        const int r = rb * 16 + g8;
                        yb[(size_t)r * kTe + 2 * t4] = yp[0];
                        yb[(size_t)r * kTe + 2 * t4 + 1] = yp[1];
                        yb[(size_t)(r + 8) * kTe + 2 * t4] = yp[2];
                        yb[(size_t)(r + 8) * kTe + 2 * t4 + 1] = yp[3];
                        if (m > 0) {
                            yb[(size_t)(nm + r) * kTe + 2 * t4] = ym[0];
                            yb[(size_t)(nm + r) * kTe + 2 * t4 + 1] = ym[1];
                            yb[(size_t)(nm + r + 8) * kTe + 2 * t4] = ym[2];
                            yb[(size_t)(nm + r + 8) * kTe + 2 * t4 + 1] = ym[3];
                        }
                    }
                    // D G_i rows of the block (unscaled)
                    for (int t = tid; t < nm * kTe; t += nt) {
                        const int r = t / kTe, e = t % kTe;
                        const int l3 = m + r / C, c = r % C, w3 = 2 * l3 + 1;
                        float gp = 0.f, gm = 0.f;
                        if (e < ne) {
                            const float* gi = Gi + (size_t)(l3 * l3) * C + c;
                            float dp_[kPRow], dm_[kPRow];
                            ld_row(Dm + e * WP + kPRow * (l3 * l3 + l3 + m), dp_);
                            ld_row(Dm + e * WP + kPRow * (l3 * l3 + l3 - m), dm_);
#pragma unroll
                            for (int n = 0; n < 2 * L + 1; ++n) {
                                const float gv = (n < w3) ? gi[(size_t)n * C] : 0.f;
                                gp = fmaf(dp_[n], gv, gp);
                                gm = fmaf(dm_[n], gv, gm);
                            }
                        }
                        gy[(size_t)r * kTe + e] = gp;
                        if (m > 0) gy[(size_t)(nm + r) * kTe + e] = gm;
                    }
                }
                for (int r = tid; r < (TC ? 0 : nm); r += nt) {
                    const int l3 = m + r / C, c = r % C;
                    float op[kTe], om[kTe];
#pragma unroll
                    for (int e = 0; e < kTe; ++e) { op[e] = 0.f; om[e] = 0.f; }
                    for (int kk = 0; kk < nm; ++kk) {
                        const float a = At[(size_t)kk * nm + r];
                        const float4* hp = reinterpret_cast<const float4*>(hs + (size_t)kk * kTe);
                        if (m == 0) {
#pragma unroll
                            for (int q4 = 0; q4 < kTe / 4; ++q4) {
                                const float4 v = hp[q4];
                                op[4 * q4 + 0] = fmaf(a, v.x, op[4 * q4 + 0]);
                                op[4 * q4 + 1] = fmaf(a, v.y, op[4 * q4 + 1]);
                                op[4 * q4 + 2] = fmaf(a, v.z, op[4 * q4 + 2]);
                                op[4 * q4 + 3] = fmaf(a, v.w, op[4 * q4 + 3]);
                            }
                        } else {
                            const float b = Bt[(size_t)kk * nm + r];
                            const float4* hmn = reinterpret_cast<const float4*>(hs + (size_t)(nm + kk) * kTe);
#pragma unroll
                            for (int q4 = 0; q4 < kTe / 4; ++q4) {
                                const float4 u = hp[q4], v = hmn[q4];
                                op[4 * q4 + 0] = fmaf(a, u.x, fmaf(-b, v.x, op[4 * q4 + 0]));
                                op[4 * q4 + 1] = fmaf(a, u.y, fmaf(-b, v.y, op[4 * q4 + 1]));
                                op[4 * q4 + 2] = fmaf(a, u.z, fmaf(-b, v.z, op[4 * q4 + 2]));
                                op[4 * q4 + 3] = fmaf(a, u.w, fmaf(-b, v.w, op[4 * q4 + 3]));
                                om[4 * q4 + 0] = fmaf(b, u.x, fmaf(a, v.x, om[4 * q4 + 0]));
                                om[4 * q4 + 1] = fmaf(b, u.y, fmaf(a, v.y, om[4 * q4 + 1]));
                                om[4 * q4 + 2] = fmaf(b, u.z, fmaf(a, v.z, om[4 * q4 + 2]));
                                om[4 * q4 + 3] = fmaf(b, u.w, fmaf(a, v.w, om[4 * q4 + 3]));
                            }
                        }
                    }
                    const int w3 = 2 * l3 + 1;
                    const float* gi = Gi + (size_t)(l3 * l3) * C + c;
#pragma unroll
                    for (int e = 0; e < kTe; ++e) {
                        float gp = 0.f, gm = 0.f;
                        if (e < ne) {
                            const float* Dp_ = Dm + e * WP + kPRow * (l3 * l3 + l3 + m);
                            const float* Dn_ = Dm + e * WP + kPRow * (l3 * l3 + l3 - m);
                            for (int n = 0; n < w3; ++n) {
                                const float gv = gi[(size_t)n * C];
                                gp = fmaf(Dp_[n], gv, gp);
                                gm = fmaf(Dn_[n], gv, gm);
                            }
                        }
                        gy[(size_t)r * kTe + e] = gp;
                        yb[(size_t)r * kTe + e] = op[e];
                        if (m > 0) {
                            gy[(size_t)(nm + r) * kTe + e] = gm;
                            yb[(size_t)(nm + r) * kTe + e] = om[e];
                        }
                    }
                }
                __syncthreads();
                // beta^h = <D G_i, Y> over the head's rows, and the first direction term
                // alpha <dD_a G_i, Y>: one warp per (edge, head), lanes over the rows
                const int rows_h = (L + 1 - m) * dh;
                for (int task = warp; task < ne * H; task += nt / 32) {
                    const int e = task / H, h = task % H;
                    const float* Ex = Dx + e * WP;
                    const float* Ey = Dy + e * WP;
                    float bs = 0.f, tx = 0.f, ty = 0.f;
                    for (int q = lane; q < rows_h; q += 32) {
                        const int l3 = m + q / dh, c = h * dh + q % dh, w3 = 2 * l3 + 1;
                        const int r = (l3 - m) * C + c;
                        const float* gi = Gi + (size_t)(l3 * l3) * C + c;
                        const int op_ = kPRow * (l3 * l3 + l3 + m), om_ = kPRow * (l3 * l3 + l3 - m);
                        float gr_[2 * L + 1];
#pragma unroll
                        for (int n = 0; n < 2 * L + 1; ++n) gr_[n] = (n < w3) ? gi[(size_t)n * C] : 0.f;
                        float ra[kPRow], rb_[kPRow];
                        float xp = 0.f, xm = 0.f, zp = 0.f, zm = 0.f;
                        ld_row(Ex + op_, ra);
                        ld_row(Ey + op_, rb_);
#pragma unroll
                        for (int n = 0; n < 2 * L + 1; ++n) {
                            xp = fmaf(ra[n], gr_[n], xp);
                            zp = fmaf(rb_[n], gr_[n], zp);
                        }
                        if (m > 0) {
                            ld_row(Ex + om_, ra);
                            ld_row(Ey + om_, rb_);
#pragma unroll
                            for (int n = 0; n < 2 * L + 1; ++n) {
                                xm = fmaf(ra[n], gr_[n], xm);
                                zm = fmaf(rb_[n], gr_[n], zm);
                            }
                        }
                        const float yp = yb[(size_t)r * kTe + e];
                        bs = fmaf(gy[(size_t)r * kTe + e], yp, bs);
                        tx = fmaf(xp, yp, tx);
                        ty = fmaf(zp, yp, ty);
                        if (m > 0) {
                            const float ym = yb[(size_t)(nm + r) * kTe + e];
                            bs = fmaf(gy[(size_t)(nm + r) * kTe + e], ym, bs);
                            tx = fmaf(xm, ym, tx);
                            ty = fmaf(zm, ym, ty);
                        }
                    }
                    bs = warp_sum(bs);
                    tx = warp_sum(tx);
                    ty = warp_sum(ty);
                    if (lane == 0) {
                        const float al = alpha[e * H + h];
                        beta[e * H + h] += bs;
                        atomicAdd(&geo[e * 12 + 10], al * tx);
                        atomicAdd(&geo[e * 12 + 11], al * ty);
                    }
                }
                __syncthreads();
                // dY = alpha D G_i
                for (int t = tid; t < (m > 0 ? 2 : 1) * nm * kTe; t += nt) {
                    const int rr = t / kTe, e = t % kTe;
                    const int c = (rr % nm) % C;
                    const float v = gy[t] * alpha[e * H + c / dh];
                    gy[t] = v;
                    if constexpr (TC) gy16[(size_t)((rr / nm) * kTe + e) * np + rr % nm] = __float2half_rn(v);
                }
                __syncthreads();
                if constexpr (TC) {
                    // dX+ = A^T dY+ + B^T dY-, dX- = -B^T dY+ + A^T dY-: one warp per 16 columns,
                    // into the Y buffer (Y is no longer needed) as [s][column][edge]
                    const __half* At16 = P.wt16 + so2_offset(L, C, m, 0);
                    const __half* Bt16 = P.wt16 + so2_offset(L, C, m, 1);
                    for (int cb = warp; cb < nm / 16; cb += nwarp) {
                        float dxp[4] = {0.f, 0.f, 0.f, 0.f}, dxm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                        for (int r0 = 0; r0 < nm; r0 += 16) {
                            const size_t fo = (((size_t)cb * (nm >> 4) + (r0 >> 4)) * 32 + lane) * 8;
                            uint32_t aa[4];
                            *reinterpret_cast<uint4*>(aa) = *reinterpret_cast<const uint4*>(At16 + fo);
                            const __half* yp = gy16 + (size_t)g8 * np + r0 + 2 * t4;
                            const uint32_t yp0 = *reinterpret_cast<const uint32_t*>(yp);
                            const uint32_t yp1 = *reinterpret_cast<const uint32_t*>(yp + 8);
                            mma16816(dxp, aa, yp0, yp1);
                            if (m > 0) {
                                uint32_t ab[4], an[4];
                                *reinterpret_cast<uint4*>(ab) = *reinterpret_cast<const uint4*>(Bt16 + fo);
#pragma unroll
                                for (int q = 0; q < 4; ++q) an[q] = ab[q] ^ 0x80008000u;
                                const __half* ym = gy16 + (size_t)(kTe + g8) * np + r0 + 2 * t4;
                                const uint32_t ym0 = *reinterpret_cast<const uint32_t*>(ym);
                                const uint32_t ym1 = *reinterpret_cast<const uint32_t*>(ym + 8);
                                mma16816(dxp, ab, ym0, ym1);
                                mma16816(dxm, an, yp0, yp1);
                                mma16816(dxm, aa, ym0, ym1);
                            }
                        }
                        const int k = cb * 16 + g8;
                        yb[(size_t)k * kTe + 2 * t4] = dxp[0];
                        yb[(size_t)k * kTe + 2 * t4 + 1] = dxp[1];
                        yb[(size_t)(k + 8) * kTe + 2 * t4] = dxp[2];
                        yb[(size_t)(k + 8) * kTe + 2 * t4 + 1] = dxp[3];
                        if (m > 0) {
                            yb[(size_t)(nm + k) * kTe + 2 * t4] = dxm[0];
                            yb[(size_t)(nm + k) * kTe + 2 * t4 + 1] = dxm[1];
                            yb[(size_t)(nm + k + 8) * kTe + 2 * t4] = dxm[2];
                            yb[(size_t)(nm + k + 8) * kTe + 2 * t4 + 1] = dxm[3];
                        }
                    }
                    __syncthreads();
                }
                // dX~ = F^T(dY) column by column, and what it feeds: dx_j, dg_v, the second direction term
                const size_t oa = so2_offset(L, C, m, 0), ob = so2_offset(L, C, m, 1);
                float t2x[kTe], t2y[kTe];
#pragma unroll
                for (int e = 0; e < kTe; ++e) { t2x[e] = 0.f; t2y[e] = 0.f; }
                for (int kc = tid; kc < nm; kc += nt) {
                    const int l1 = m + kc / C, c = kc % C;
                    float dp[kTe], dq[kTe];
#pragma unroll
                    for (int e = 0; e < kTe; ++e) {
                        dp[e] = TC ? yb[(size_t)kc * kTe + e] : 0.f;
                        dq[e] = (TC && m > 0) ? yb[(size_t)(nm + kc) * kTe + e] : 0.f;
                    }
                    for (int r = 0; r < (TC ? 0 : nm); ++r) {
                        const float a = load_feat(W, oa + (size_t)r * nm + kc);
                        const float4* yp4 = reinterpret_cast<const float4*>(gy + (size_t)r * kTe);
                        if (m == 0) {
#pragma unroll
                            for (int q4 = 0; q4 < kTe / 4; ++q4) {
                                const float4 v = yp4[q4];
                                dp[4 * q4 + 0] = fmaf(a, v.x, dp[4 * q4 + 0]);
                                dp[4 * q4 + 1] = fmaf(a, v.y, dp[4 * q4 + 1]);
                                dp[4 * q4 + 2] = fmaf(a, v.z, dp[4 * q4 + 2]);
                                dp[4 * q4 + 3] = fmaf(a, v.w, dp[4 * q4 + 3]);
                            }
                        } else {
                            const float b = load_feat(W, ob + (size_t)r * nm + kc);
                            const float4* ym4 = reinterpret_cast<const float4*>(gy + (size_t)(nm + r) * kTe);
#pragma unroll
                            for (int q4 = 0; q4 < kTe / 4; ++q4) {
                                const float4 u = yp4[q4], v = ym4[q4];
                                dp[4 * q4 + 0] = fmaf(a, u.x, fmaf(b, v.x, dp[4 * q4 + 0]));
                                dp[4 * q4 + 1] = fmaf(a, u.y, fmaf(b, v.y, dp[4 * q4 + 1]));
                                dp[4 * q4 + 2] = fmaf(a, u.z, fmaf(b, v.z, dp[4 * q4 + 2]));
                                dp[4 * q4 + 3] = fmaf(a, u.w, fmaf(b, v.w, dp[4 * q4 + 3]));
                                dq[4 * q4 + 0] = fmaf(-b, u.x, fmaf(a, v.x, dq[4 * q4 + 0]));
                                dq[4 * q4 + 1] = fmaf(-b, u.y, fmaf(a, v.y, dq[4 * q4 + 1]));
                                dq[4 * q4 + 2] = fmaf(-b, u.z, fmaf(a, v.z, dq[4 * q4 + 2]));
                                dq[4 * q4 + 3] = fmaf(-b, u.w, fmaf(a, v.w, dq[4 * q4 + 3]));
                            }
                        }
                    }
                    const int w1 = 2 * l1 + 1;
#pragma unroll
                    for (int e = 0; e < kTe; ++e) {
                        if (e < ne) {
                            const int pp = e * WP + kPRow * (l1 * l1 + l1 + m), pm = e * WP + kPRow * (l1 * l1 + l1 - m);
                            const size_t xb = ((size_t)jn[e] * K + l1 * l1) * C + c;
                            const float gv = g[e * G + l1 * C + c];
                            float rp = 0.f, rm = 0.f, xp = 0.f, xm = 0.f, zp = 0.f, zm = 0.f;
                            float xr[2 * L + 1];  // all loads issued before the arithmetic
#pragma unroll
                            for (int n = 0; n < 2 * L + 1; ++n)
                                xr[n] = (n < w1) ? load_feat(x, xb + (size_t)n * C) : 0.f;
                            float ra[kPRow], rb_[kPRow];
                            ld_row(Dm + pp, ra);
                            ld_row(Dm + pm, rb_);
#pragma unroll
                            for (int n = 0; n < 2 * L + 1; ++n) {
                                rp = fmaf(ra[n], xr[n], rp);
                                rm = fmaf(rb_[n], xr[n], rm);
                                if (n < w1) {
                                    float gxv = ra[n] * dp[e];
                                    if (m > 0) gxv = fmaf(rb_[n], dq[e], gxv);
                                    atomicAdd(P.gx + xb + (size_t)n * C, gv * gxv);
                                }
                            }
                            ld_row(Dx + pp, ra);
                            ld_row(Dx + pm, rb_);
#pragma unroll
                            for (int n = 0; n < 2 * L + 1; ++n) {
                                xp = fmaf(ra[n], xr[n], xp);
                                xm = fmaf(rb_[n], xr[n], xm);
                            }
                            ld_row(Dy + pp, ra);
                            ld_row(Dy + pm, rb_);
#pragma unroll
                            for (int n = 0; n < 2 * L + 1; ++n) {
                                zp = fmaf(ra[n], xr[n], zp);
                                zm = fmaf(rb_[n], xr[n], zm);
                            }
                            float dg = dp[e] * rp, tx = dp[e] * xp, ty = dp[e] * zp;
                            if (m > 0) {
                                dg = fmaf(dq[e], rm, dg);
                                tx = fmaf(dq[e], xm, tx);
                                ty = fmaf(dq[e], zm, ty);
                            }
                            dgv[e * Gv + l1 * C + c] += dg;
                            t2x[e] = fmaf(gv, tx, t2x[e]);
                            t2y[e] = fmaf(gv, ty, t2y[e]);
                        }
                    }
                }
#pragma unroll
                for (int e = 0; e < kTe; ++e) {
                    const float sx = warp_sum(t2x[e]), sy = warp_sum(t2y[e]);
                    if (lane == 0 && e < ne) {
                        atomicAdd(&geo[e * 12 + 10], sx);
                        atomicAdd(&geo[e * 12 + 11], sy);
                    }
                }
                __syncthreads();
            }
            // value gates -> rho: dLoss/drho_k = sum_c W_rad[k][c] dg_v[c]; dW_rad += rho (x) dg_v
            for (int pk = warp; pk < kTe * nr; pk += nt / 32) {
                const int e = pk / nr, kb = pk % nr;
                float s = 0.f;
                for (int c = lane; c < Gv; c += 32) s = fmaf(P.Wrad[(size_t)kb * G + c], dgv[e * Gv + c], s);
                s = warp_sum(s);
                if (lane == 0) red[pk] = s;
            }
            for (int t = tid; t < nr * Gv; t += nt) {
                const int kb = t / Gv, c = t % Gv;
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < kTe; ++e) s = fmaf(rho[e * nr + kb], dgv[e * Gv + c], s);
                gWr[(size_t)kb * G + c] += s;
            }
            __syncthreads();
            if (tid < ne) {
                const int e = tid;
                const float* gg = geo + e * 12;
                float dd = 0.f;
                for (int kb = 0; kb < nr; ++kb) dd = fmaf(rhop[e * nr + kb], red[e * nr + kb], dd);
                const float id = 1.f / gg[3];
                const int j = jn[e];
#pragma unroll
                for (int c = 0; c < 3; ++c) {
                    const float dr = dd * gg[c] + (gg[10] * gg[4 + c] + gg[11] * gg[7 + c]) * id;
                    atomicAdd(P.gpos + 3 * (size_t)j + c, dr);
                    atomicAdd(gpi + c, -dr);
                }
                for (int h = 0; h < H; ++h) {
                    P.beta[(size_t)(e0 + e) * H + h] = beta[e * H + h];
                    atomicAdd(dlt + h, alpha[e * H + h] * beta[e * H + h]);
                }
            }
            __syncthreads();
        }
        // logit gradient: needs delta_i over all the node's edges
        {
            const int h = tid % H;
            const float* qi = P.q + (size_t)i * C + h * dh;
            for (int e = tid / H; e < deg; e += nt / H) {
                const int j = P.col[e_begin + e];
                float3 u;
                float d, gap;
                const Logit lg = edge_logit(P, i, j, h, Gv, G, inv, &u, &d, &gap);
                const float al = expf(lg.a - lse_s[h]);
                const float da = al * (P.beta[(size_t)(e_begin + e) * H + h] - dlt[h]);
                const float dga = da * lg.dot * inv, ds = da * lg.ga * inv;
                const float* kj = P.k + (size_t)j * C + h * dh;
                for (int c = 0; c < dh; ++c) {
                    atomicAdd(gqi + h * dh + c, ds * kj[c]);
                    atomicAdd(P.gk + (size_t)j * C + h * dh + c, ds * qi[c]);
                }
                for (int kb = 0; kb < nr; ++kb) {
                    float v, dv;
                    rbf_and_deriv(d, kb, P.cutoff, nr, v, dv);
                    atomicAdd(gWr + (size_t)kb * G + Gv + h, v * dga);
                }
                const float dd = dga * gap;
                atomicAdd(P.gpos + 3 * (size_t)j + 0, dd * u.x);
                atomicAdd(P.gpos + 3 * (size_t)j + 1, dd * u.y);
                atomicAdd(P.gpos + 3 * (size_t)j + 2, dd * u.z);
                atomicAdd(gpi + 0, -dd * u.x);
                atomicAdd(gpi + 1, -dd * u.y);
                atomicAdd(gpi + 2, -dd * u.z);
            }
        }
        __syncthreads();
        for (int c = tid; c < C; c += nt) P.gq[(size_t)i * C + c] = gqi[c];
        if (tid < 3) atomicAdd(P.gpos + 3 * (size_t)i + tid, gpi[tid]);
    }
    __syncthreads();
    for (int t = tid; t < nr * G; t += nt) atomicAdd(P.gWrad + t, gWr[t]);
}

// dW_so2 = sum over edges of dY (x) X~, one 128 x 64 tile (rows x columns) of
// one |m| block per CTA (A and B tiles together for m >= 1), over one of
// kDwSplit edge ranges:
//   dA += dY+ X~+^T + dY- X~-^T,   dB += dY- X~+^T - dY+ X~-^T
// with dY(l3, +-m, c) = alpha^{head c} sum_n D^l3[+-m][n] G_i[l3, n, c] and
// X~(l1, +-m, c) = g_v[l1, c] sum_n D^l1[+-m][n] x_j[l1, n, c], rebuilt per
// edge from the geometry (no per-edge storage). Edges are visited in CSR
// order in chunks of kDwChunk (one thread per edge for the frame and weights),
// then in sub-chunks of kDwE for the operands.
__device__ __forceinline__ int drow_off(int m, int l, int s) {
    // rows (l+m) and (l-m) of D^l for l = m..L, stored per edge back to back
    const int nrow = (m == 0) ? 1 : 2;
    int o = 0;
    for (int k = m; k < l; ++k) o += nrow * (2 * k + 1);
    return o + s * (2 * l + 1);
}

size_t dw_part_floats(int L, int C, int M) { return (size_t)kDwSplit * so2_total(L, C, M); }

size_t dw_smem_bytes(int H, int n_rbf) {
    return 4 * ((size_t)kDwChunk * 50 + (size_t)kDwChunk * n_rbf + (size_t)kDwChunk * H + 2 * kDwChunk +
                (size_t)n_rbf * kDwC + 2ull * kDwE * (kDwR + kDwC));
}

int n_dw_tiles(int L, int C, int M) {
    int n = 0;
    for (int m = 0; m <= M; ++m) {
        const int nm = (L + 1 - m) * C;
        n += ((nm + kDwR - 1) / kDwR) * ((nm + kDwC - 1) / kDwC);
    }
    return n;
}

// fp32 storage: fp32 operands and FMA accumulation (thread tile 8 x 4).
template <int L, typename T>
__global__ void __launch_bounds__(kNt, 2) k_bwd_dw(BwdParams P) {
    constexpr int K = n_sh(L);
    constexpr int WS = wig_size(L);
    const int C = P.C, H = P.H, dh = C / H, nr = P.n_rbf;
    const int Gv = (L + 1) * C, G = Gv + H;
    const T* __restrict__ x = static_cast<const T*>(P.x);
    // this CTA's tile (blocks m = 0..M in order, tiles of a block row-major) and edge range
    const int split = blockIdx.x / P.dw_tiles;
    int m = 0, nm = (L + 1) * C, b = blockIdx.x % P.dw_tiles;
    int sr = (nm + kDwR - 1) / kDwR, sc = (nm + kDwC - 1) / kDwC;
    while (b >= sr * sc && m < P.M) {
        b -= sr * sc;
        ++m;
        nm = (L + 1 - m) * C;
        sr = (nm + kDwR - 1) / kDwR;
        sc = (nm + kDwC - 1) / kDwC;
    }
    const int r0 = (b / sc) * kDwR, k0 = (b % sc) * kDwC;
    const int nrow = (m == 0) ? 1 : 2;

    extern __shared__ float sm[];
    float* drow = sm;                          // [chunk][50]
    float* rho = drow + kDwChunk * 50;         // [chunk][nr]
    float* alpha = rho + kDwChunk * nr;        // [chunk][H]
    int* ei = reinterpret_cast<int*>(alpha + kDwChunk * H);  // [chunk] node i
    int* ej = ei + kDwChunk;                   // [chunk] neighbour j
    float* wr = reinterpret_cast<float*>(ej + kDwChunk);     // [nr][kDwC] W_rad columns of the tile
    float* Yop = wr + nr * kDwC;               // [2][kDwE][kDwR] dY rows of the tile
    float* Xop = Yop + 2 * kDwE * kDwR;        // [2][kDwE][kDwC] X~ columns of the tile

    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const float inv = rsqrtf((float)dh);
    float accA[8][4], accB[8][4];  // [row][col] of this thread's 8 x 4 part of the tile
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) { accA[a][c] = 0.f; accB[a][c] = 0.f; }

    for (int t = tid; t < nr * kDwC; t += kNt) {
        const int kb = t / kDwC, kx = k0 + t % kDwC;
        wr[t] = (kx < nm) ? P.Wrad[(size_t)kb * G + (m + kx / C) * C + kx % C] : 0.f;
    }
    // this thread's operand roles (fixed for the CTA): dY row (sign y_s, row y_q) and X~ column
    // (sign x_s, column x_q, edges of parity x_half); offsets into a node's [K][C] row, into
    // an edge's Wigner rows, the degree's width and the head
    const int y_s = tid / kDwR, y_q = tid % kDwR, ry = r0 + y_q;
    const bool y_ok = y_s < nrow && ry < nm;
    const int y_l = m + (y_ok ? ry / C : 0), y_c = y_ok ? ry % C : 0;
    const int y_g = y_l * y_l * C + y_c, y_w = 2 * y_l + 1, y_d = y_ok ? drow_off(m, y_l, y_s) : 0;
    const int y_h = y_c / dh;
    const int x_role = tid % (2 * kDwC), x_half = tid / (2 * kDwC);
    const int x_s = x_role / kDwC, x_q = x_role % kDwC, kxx = k0 + x_q;
    const bool x_ok = x_s < nrow && kxx < nm;
    const int x_l = m + (x_ok ? kxx / C : 0), x_c = x_ok ? kxx % C : 0;
    const int x_g = x_l * x_l * C + x_c, x_w = 2 * x_l + 1, x_d = x_ok ? drow_off(m, x_l, x_s) : 0;
    static_assert(2 * kDwR == kNt && 4 * kDwC == kNt, "operand roles: one dY row per thread, two threads per X~ column");

    const int e_lo = (int)((long long)P.n_pairs * split / kDwSplit);
    const int e_hi = (int)((long long)P.n_pairs * (split + 1) / kDwSplit);
    for (int c0 = e_lo; c0 < e_hi; c0 += kDwChunk) {
        const int nc = min(kDwChunk, e_hi - c0);
        __syncthreads();
        if (tid < nc) {
            const int e = c0 + tid;
            int lo = 0, hi = P.n_atoms - 1;  // node i: last n with row_ptr[n] <= e
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (P.row_ptr[mid] <= e) lo = mid; else hi = mid - 1;
            }
            const int i = lo, j = P.col[e];
            ei[tid] = i;
            ej[tid] = j;
            const float3 r = edge_vec(P.pos, i, j, P.box);
            const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
            float R[3][3];
            edge_frame(r.x / d, r.y / d, r.z / d, R);
            float D[WS];
            wigner_blocks<L>(R, D);
            float* dr = drow + tid * 50;
            for (int l = m; l <= L; ++l) {
                const int w = 2 * l + 1;
                for (int s2 = 0; s2 < nrow; ++s2) {
                    const int row = s2 == 0 ? l + m : l - m;
                    for (int n = 0; n < w; ++n) dr[drow_off(m, l, s2) + n] = D[wig_off(l) + row * w + n];
                }
            }
            for (int kb = 0; kb < nr; ++kb) rho[tid * nr + kb] = rbf(d, kb, P.cutoff, nr);
            for (int h = 0; h < H; ++h) {
                float ga = 0.f;
                for (int kb = 0; kb < nr; ++kb) ga = fmaf(rho[tid * nr + kb], P.Wrad[(size_t)kb * G + Gv + h], ga);
                const float* qi = P.q + (size_t)i * C + h * dh;
                const float* kj = P.k + (size_t)j * C + h * dh;
                float dot = 0.f;
                for (int c = 0; c < dh; ++c) dot = fmaf(qi[c], kj[c], dot);
                alpha[tid * H + h] = expf(ga * dot * inv - P.lse[(size_t)i * H + h]);
            }
        }
        __syncthreads();
        for (int s0 = 0; s0 < nc; s0 += kDwE) {
            const int ns = min(kDwE, nc - s0);
            // operands of the sub-chunk: dY rows r0.. (thread = one (sign, row)), X~ columns
            // k0.. (thread = one (sign, column) and every other edge); G_i stays in registers
            // while consecutive edges share their node
            {
                int cached = -1;
                float gr[2 * L + 1];
#pragma unroll
                for (int n = 0; n < 2 * L + 1; ++n) gr[n] = 0.f;
                for (int e = 0; e < kDwE; ++e) {
                    float v = 0.f;
                    if (e < ns && y_ok) {
                        const int el = s0 + e, node = ei[el];
                        if (node != cached) {
                            const float* gi = P.G + (size_t)node * K * C + y_g;
#pragma unroll
                            for (int n = 0; n < 2 * L + 1; ++n) gr[n] = (n < y_w) ? gi[(size_t)n * C] : 0.f;
                            cached = node;
                        }
                        const float* dr = drow + el * 50 + y_d;
                        float acc = 0.f;
#pragma unroll
                        for (int n = 0; n < 2 * L + 1; ++n)
                            if (n < y_w) acc = fmaf(dr[n], gr[n], acc);
                        v = alpha[el * H + y_h] * acc;
                    }
                    Yop[(y_s * kDwE + e) * kDwR + y_q] = v;
                }
                for (int e = x_half; e < kDwE; e += 2) {
                    float v = 0.f;
                    if (e < ns && x_ok) {
                        const int el = s0 + e;
                        const size_t xb = (size_t)ej[el] * K * C + x_g;
                        float xr[2 * L + 1];  // all loads issued before the arithmetic
#pragma unroll
                        for (int n = 0; n < 2 * L + 1; ++n) xr[n] = (n < x_w) ? load_feat(x, xb + (size_t)n * C) : 0.f;
                        const float* dr = drow + el * 50 + x_d;
                        float acc = 0.f;
#pragma unroll
                        for (int n = 0; n < 2 * L + 1; ++n)
                            if (n < x_w) acc = fmaf(dr[n], xr[n], acc);
                        float gv = 0.f;
                        for (int kb = 0; kb < nr; ++kb) gv = fmaf(rho[el * nr + kb], wr[kb * kDwC + x_q], gv);
                        v = gv * acc;
                    }
                    Xop[(x_s * kDwE + e) * kDwC + x_q] = v;
                }
            }
            __syncthreads();
            {
                for (int e = 0; e < ns; ++e) {
                    const float4 y0 = *reinterpret_cast<const float4*>(Yop + e * kDwR + ty * 8);
                    const float4 y1 = *reinterpret_cast<const float4*>(Yop + e * kDwR + ty * 8 + 4);
                    const float4 xv = *reinterpret_cast<const float4*>(Xop + e * kDwC + tx * 4);
                    const float ypa[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
                    const float xpa[4] = {xv.x, xv.y, xv.z, xv.w};
                    if (m == 0) {
#pragma unroll
                        for (int a = 0; a < 8; ++a)
#pragma unroll
                            for (int c = 0; c < 4; ++c) accA[a][c] = fmaf(ypa[a], xpa[c], accA[a][c]);
                    } else {
                        const float4 z0 = *reinterpret_cast<const float4*>(Yop + (kDwE + e) * kDwR + ty * 8);
                        const float4 z1 = *reinterpret_cast<const float4*>(Yop + (kDwE + e) * kDwR + ty * 8 + 4);
                        const float4 xw = *reinterpret_cast<const float4*>(Xop + (kDwE + e) * kDwC + tx * 4);
                        const float yma[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
                        const float xma[4] = {xw.x, xw.y, xw.z, xw.w};
#pragma unroll
                        for (int a = 0; a < 8; ++a)
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                accA[a][c] = fmaf(ypa[a], xpa[c], fmaf(yma[a], xma[c], accA[a][c]));
                                accB[a][c] = fmaf(yma[a], xpa[c], fmaf(-ypa[a], xma[c], accB[a][c]));
                            }
                    }
                }
            }
            __syncthreads();
        }
    }
    const size_t oa = so2_offset(L, C, m, 0), ob = so2_offset(L, C, m, 1);
    float* dst = P.gWpart + (size_t)split * so2_total(L, C, P.M);
    {
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int r = r0 + ty * 8 + a;
            if (r >= nm) continue;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int kx = k0 + tx * 4 + c;
                if (kx >= nm) continue;
                dst[oa + (size_t)r * nm + kx] = accA[a][c];
                if (m > 0) dst[ob + (size_t)r * nm + kx] = accB[a][c];
            }
        }
    }
}

constexpr int kURbf = 32;  // radial basis per edge, padded (n_rbf <= 32)

// Position of element (r, k) of an n x n block (n a multiple of 16) in fragment
// order: 16 x 16 tiles row-major, and within a tile the 8 halves that lane
// (g, t) of an m16n8k16 A fragment holds, in register order
// (r g, k 2t..2t+1), (r g+8, k 2t..), (r g, k 2t+8..), (r g+8, k 2t+8..).
__host__ __device__ inline size_t frag_pos(int r, int k, int n) {
    const int rb = r >> 4, kb = k >> 4, rr = r & 15, kk = k & 15;
    const int lane = (rr & 7) * 4 + ((kk & 7) >> 1), q = (rr >> 3) + 2 * (kk >> 3);
    return (((size_t)rb * (n >> 4) + kb) * 32 + lane) * 8 + q * 2 + (kk & 1);
}

// Packed SO(2) weights -> fp16 in fragment order: each block (w16) and each
// block transposed (wt16), so an A fragment is one 16-byte load per lane
template <typename T>
__global__ void k_bwd_w16(const T* __restrict__ w, int L, int C, int M, __half* w16, __half* wt16) {
    const size_t total = so2_total(L, C, M);
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        size_t off = 0;
        int n = (L + 1) * C, blk = 0;
        while (e >= off + (size_t)n * n) {
            off += (size_t)n * n;
            ++blk;
            n = (L + 1 - (blk + 1) / 2) * C;
        }
        const size_t loc = e - off;
        const int r = (int)(loc / n), k = (int)(loc % n);
        const __half v = __float2half_rn(load_feat(w, e));
        w16[off + frag_pos(r, k, n)] = v;
        wt16[off + frag_pos(k, r, n)] = v;
    }
}

// gW = the edge-range partial sums, added in a fixed order
__global__ void k_bwd_dw_sum(const float* __restrict__ part, size_t total, float* out) {
    for (size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (size_t)gridDim.x * blockDim.x) {
        float s = part[t];
        for (int k = 1; k < kDwSplit; ++k) s += part[(size_t)k * total + t];
        out[t] = s;
    }
}

// dW_q = sum_i dq_i (x) x_i[l=0], dW_k likewise (q = W_q x[l=0]); one thread per weight
template <typename T>
__global__ void k_bwd_wqk(const T* __restrict__ x, int n, int K, int C, const float* __restrict__ gq,
                          const float* __restrict__ gk, float* gWq, float* gWk) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= C * C) return;
    const int o = t / C, c = t % C;
    float sq = 0.f, sk = 0.f;
    for (int i = 0; i < n; ++i) {
        const float xv = load_feat(x, (size_t)i * K * C + c);
        sq = fmaf(gq[(size_t)i * C + o], xv, sq);
        sk = fmaf(gk[(size_t)i * C + o], xv, sk);
    }
    if (gWq) gWq[t] = sq;
    if (gWk) gWk[t] = sk;
}

// dx[i, l=0, c] += sum_o W_q[o][c] dq_i[o] + W_k[o][c] dk_i[o]
__global__ void k_bwd_x0(int n, int K, int C, const float* __restrict__ Wq, const float* __restrict__ Wk,
                         const float* __restrict__ gq, const float* __restrict__ gk, float* gx) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n * C) return;
    const int i = t / C, c = t % C;
    float s = 0.f;
    for (int o = 0; o < C; ++o) {
        s = fmaf(Wq[(size_t)o * C + c], gq[(size_t)i * C + o], s);
        s = fmaf(Wk[(size_t)o * C + c], gk[(size_t)i * C + o], s);
    }
    gx[(size_t)i * K * C + c] += s;
}

template <int L, typename T>
cudaError_t launch_node(const BwdParams& P, size_t smem, int grid, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(k_bwd_node<L, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    k_bwd_node<L, T><<<grid, kNodeNt, smem, s>>>(P);
    return cudaGetLastError();
}

template <int L, typename T>
cudaError_t launch_dw(const BwdParams& P, int n_tiles, size_t smem, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(k_bwd_dw<L, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    k_bwd_dw<L, T><<<n_tiles, kNt, smem, s>>>(P);
    return cudaGetLastError();
}



// ---------------------------------------------------------------------------
// SO(2) weight gradient for bf16 storage as GEMMs over the edges. Per chunk of
// edges, k_bwd_ops writes each edge's two operand rows in fp16:
//   X[e][col(l1, m) + c] = g_v(d_e)[l1, c] sum_n D_e^{l1}[l1 + m][n] x_j[l1, n][c]
//       (the rotated, gated neighbour features the maps act on),
//   Y[e][col(l3, m) + c] = alpha_e^{head(c)} sum_n D_e^{l3}[l3 + m][n] G_i[l3, n][c]
//       (the softmax-weighted upstream gradient in the edge frame, dLoss/dY),
// for m = 0 and m = +-mu (mu <= M), in the packed order of the SO(2) blocks:
// block mu holds the +mu rows (l - mu) C + c, then the -mu rows (ops_col).
// The gradient of block mu is then
//   dA(mu) = sum_e Y+ X+^T + Y- X-^T,   dB(mu) = sum_e Y- X+^T - Y+ X-^T
// (dA(0) = sum_e Y0 X0^T): plain GEMMs over the chunk's edges (K = edges),
// which cuBLAS runs with fp32 accumulation into the output, chunk after chunk
// (a fixed order, so the result is deterministic). Each operand is built once
// per edge instead of once per weight tile.
constexpr int kOpsChunk = 131072;  // edges per chunk
constexpr int kOpsE = 32;         // edges per CTA of k_bwd_ops
constexpr int kOpsNt = 256;
constexpr int kOpsMaxH = 32;

__host__ __device__ inline int ops_col(int l, int m, int L, int C) {
    const int mu = m < 0 ? -m : m;
    if (mu == 0) return l * C;
    int off = (L + 1) * C;
    for (int k = 1; k < mu; ++k) off += 2 * (L + 1 - k) * C;
    const int nm = (L + 1 - mu) * C;
    return off + (m > 0 ? 0 : nm) + (l - mu) * C;
}

template <int L>
__global__ void __launch_bounds__(kOpsNt, 2) k_bwd_ops(BwdParams P, int e0, int ne, __half* __restrict__ Xo,
                                                      __half* __restrict__ Yo) {
    constexpr int K = n_sh(L), WS = wig_size(L);
    const int C = P.C, H = P.H, dh = C / H, nr = P.n_rbf, M = P.M;
    const int Gv = (L + 1) * C, G = Gv + H;
    const size_t KC = (size_t)K * C;
    const __nv_bfloat16* __restrict__ x = static_cast<const __nv_bfloat16*>(P.x);
    __shared__ float Ds[kOpsE][WS];
    __shared__ float rho[kOpsE][kURbf];
    __shared__ float alpha[kOpsE][kOpsMaxH];
    __shared__ int ei[kOpsE], ej[kOpsE];
    const int tid = threadIdx.x;
    const int eb = blockIdx.x * kOpsE;  // first edge of this CTA within the chunk
    const int nb = min(kOpsE, ne - eb);
    if (tid < nb) {
        const int e = e0 + eb + tid;
        int lo = 0, hi = P.n_atoms - 1;  // node: last n with row_ptr[n] <= e
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.row_ptr[mid] <= e) lo = mid; else hi = mid - 1;
        }
        const int i = lo, j = P.col[e];
        const float3 r = edge_vec(P.pos, i, j, P.box);
        const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
        float R[3][3];
        edge_frame(r.x / d, r.y / d, r.z / d, R);
        float D[WS];
        wigner_blocks<L>(R, D);
        for (int k2 = 0; k2 < WS; ++k2) Ds[tid][k2] = D[k2];
        float rr[kURbf];
        rbf_all<kURbf>(d, P.cutoff, nr, rr);
        for (int kb = 0; kb < kURbf; ++kb) rho[tid][kb] = rr[kb];
        const float inv = rsqrtf((float)dh);
        for (int h = 0; h < H; ++h) {
            float ga = 0.f;
            for (int kb = 0; kb < nr; ++kb) ga = fmaf(rr[kb], P.Wrad[(size_t)kb * G + Gv + h], ga);
            const float* qi = P.q + (size_t)i * C + h * dh;
            const float* kj = P.k + (size_t)j * C + h * dh;
            float dot = 0.f;
            for (int c = 0; c < dh; ++c) dot = fmaf(qi[c], kj[c], dot);
            alpha[tid][h] = expf(ga * dot * inv - P.lse[(size_t)i * H + h]);
        }
        ei[tid] = i;
        ej[tid] = j;
    }
    __syncthreads();
    const int CG = C / 8;
    for (int it = tid; it < nb * CG; it += kOpsNt) {
        const int el = it / CG, c0 = (it % CG) * 8;
        const int i = ei[el], j = ej[el];
        __half* xrow = Xo + (size_t)(eb + el) * KC;
        __half* yrow = Yo + (size_t)(eb + el) * KC;
        float al[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) al[q] = alpha[el][(c0 + q) / dh];
#pragma unroll
        for (int l = 0; l <= L; ++l) {
            constexpr int kW = 2 * L + 1;
            const int w = 2 * l + 1;
            const float* Dl = &Ds[el][wig_off(l)];
            // value gate of the 8 channels of degree l
            float gv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) gv[q] = 0.f;
            for (int kb = 0; kb < nr; ++kb) {
                const float rk = rho[el][kb];
                const float* wr = P.Wrad + (size_t)kb * G + l * C + c0;  // rows of (L+1)C + H: no vector alignment
#pragma unroll
                for (int q = 0; q < 8; ++q) gv[q] = fmaf(rk, __ldg(wr + q), gv[q]);
            }
            // X: rows (l, n) of x_j for these channels, rotated and gated
            {
                float xv[kW][8];
#pragma unroll
                for (int n = 0; n < kW; ++n) {
                    if (n < w) {
                        const uint4 u = *reinterpret_cast<const uint4*>(x + ((size_t)j * K + l * l + n) * C + c0);
                        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float2 f = __bfloat1622float2(b2[q]);
                            xv[n][2 * q] = f.x;
                            xv[n][2 * q + 1] = f.y;
                        }
                    }
                }
#pragma unroll
                for (int mu = 0; mu <= L; ++mu) {
                    if (mu > l || mu > M) continue;
#pragma unroll
                    for (int sg = 0; sg < 2; ++sg) {
                        if (mu == 0 && sg == 1) continue;
                        const int m = sg == 0 ? mu : -mu;
                        const float* Dr = Dl + (l + m) * w;  // D^l[l + m][n]
                        float o[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) o[q] = 0.f;
#pragma unroll
                        for (int n = 0; n < kW; ++n) {
                            if (n < w) {
                                const float dv = Dr[n];
#pragma unroll
                                for (int q = 0; q < 8; ++q) o[q] = fmaf(dv, xv[n][q], o[q]);
                            }
                        }
                        __align__(16) __half hx[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) hx[q] = __float2half_rn(gv[q] * o[q]);
                        *reinterpret_cast<uint4*>(xrow + ops_col(l, m, L, C) + c0) = *reinterpret_cast<const uint4*>(hx);
                    }
                }
            }
            // Y: rows (l, n) of G_i for these channels, rotated and weighted by the softmax
            {
                float gg[kW][8];
#pragma unroll
                for (int n = 0; n < kW; ++n) {
                    if (n < w) {
                        const float4* gp = reinterpret_cast<const float4*>(P.G + ((size_t)i * K + l * l + n) * C + c0);
                        const float4 ga = gp[0], gb = gp[1];
                        gg[n][0] = ga.x; gg[n][1] = ga.y; gg[n][2] = ga.z; gg[n][3] = ga.w;
                        gg[n][4] = gb.x; gg[n][5] = gb.y; gg[n][6] = gb.z; gg[n][7] = gb.w;
                    }
                }
#pragma unroll
                for (int mu = 0; mu <= L; ++mu) {
                    if (mu > l || mu > M) continue;
#pragma unroll
                    for (int sg = 0; sg < 2; ++sg) {
                        if (mu == 0 && sg == 1) continue;
                        const int m = sg == 0 ? mu : -mu;
                        const float* Dr = Dl + (l + m) * w;
                        float o[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) o[q] = 0.f;
#pragma unroll
                        for (int n = 0; n < kW; ++n) {
                            if (n < w) {
                                const float dv = Dr[n];
#pragma unroll
                                for (int q = 0; q < 8; ++q) o[q] = fmaf(dv, gg[n][q], o[q]);
                            }
                        }
                        __align__(16) __half hy[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) hy[q] = __float2half_rn(al[q] * o[q]);
                        *reinterpret_cast<uint4*>(yrow + ops_col(l, m, L, C) + c0) = *reinterpret_cast<const uint4*>(hy);
                    }
                }
            }
        }
    }
}

template <int L>
cudaError_t launch_ops(const BwdParams& P, int e0, int ne, __half* Xo, __half* Yo, cudaStream_t s) {
    count_launch();
    k_bwd_ops<L><<<(ne + kOpsE - 1) / kOpsE, kOpsNt, 0, s>>>(P, e0, ne, Xo, Yo);
    return cudaGetLastError();
}

// cuBLAS, loaded at run time (the library links no BLAS; the host process
// normally has it loaded already). One handle per CUDA context, found by the
// context's unique id, so a handle is never used in another context. Handles
// live until the process ends (a destroyed context's entry is never found
// again); the stream is set on the handle per call, so concurrent calls on
// one context from several host threads must be serialised by the caller.
struct CublasRt {
    decltype(&cublasCreate_v2) create = nullptr;
    decltype(&cublasSetStream_v2) set_stream = nullptr;
    cublasStatus_t (*gemm)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int, const void*,
                           const void*, cudaDataType, int, const void*, cudaDataType, int, const void*, void*,
                           cudaDataType, int, cublasComputeType_t, cublasGemmAlgo_t) = nullptr;
    bool ok = false;
};
CublasRt& cublas_rt() {
    static CublasRt rt;
    static std::once_flag once;
    std::call_once(once, [] {
        const char* names[] = {"libcublas.so.12", "/usr/local/cuda/lib64/libcublas.so.12", "libcublas.so"};
        void* h = nullptr;
        for (const char* n : names) {
            h = dlopen(n, RTLD_NOW | RTLD_GLOBAL);
            if (h) break;
        }
        if (!h) return;
        rt.create = reinterpret_cast<decltype(rt.create)>(dlsym(h, "cublasCreate_v2"));
        rt.set_stream = reinterpret_cast<decltype(rt.set_stream)>(dlsym(h, "cublasSetStream_v2"));
        rt.gemm = reinterpret_cast<decltype(rt.gemm)>(dlsym(h, "cublasGemmEx"));
        rt.ok = rt.create && rt.set_stream && rt.gemm;
    });
    return rt;
}
cublasHandle_t cublas_handle() {
    CublasRt& rt = cublas_rt();
    if (!rt.ok) return nullptr;
    // driver entry points through the runtime (the library does not link the driver)
    using GetCurrentFn = CUresult (*)(CUcontext*);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    if (!get_current || !get_id) {
        void* p1 = nullptr;
        void* p2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess)
            return nullptr;
        get_current = reinterpret_cast<GetCurrentFn>(p1);
        get_id = reinterpret_cast<GetIdFn>(p2);
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return nullptr;
    static std::mutex mu;
    static std::map<unsigned long long, cublasHandle_t> handles;
    std::lock_guard<std::mutex> lock(mu);
    auto it = handles.find(id);
    if (it != handles.end()) return it->second;
    cublasHandle_t h = nullptr;
    if (rt.create(&h) != CUBLAS_STATUS_SUCCESS) return nullptr;
    handles[id] = h;
    return h;
}

// out (nm x nm, row-major [f][k]) += alpha sum_e Y[e][f] X[e][k] over ne edges; X, Y point at
// the block's columns of rows of KC halves
cublasStatus_t gemm_edges(cublasHandle_t h, int nm, int ne, size_t KC, const __half* X, const __half* Y,
                          float alpha, float* out) {
    const float beta = 1.f;
    // column-major view: out^T (k x f) = X^T (k x e) * Y (e x f)
    return cublas_rt().gemm(h, CUBLAS_OP_N, CUBLAS_OP_T, nm, nm, ne, &alpha, X, CUDA_R_16F, (int)KC, Y, CUDA_R_16F,
                            (int)KC, &beta, out, CUDA_R_32F, nm, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
}

}  // namespace bwd

size_t bwd_partial_bytes(int L, int C, int M) { return 4 * bwd::dw_part_floats(L, C, M); }

size_t bwd_ops_bytes(int64_t n_pairs, int L, int C) {
    const int64_t ec = std::min<int64_t>(std::max<int64_t>(n_pairs, 1), bwd::kOpsChunk);
    return 2 * (size_t)ec * (size_t)n_sh(L) * C * 2;
}

bool bwd_supported(int L, int C, int H, int n_rbf) {
    if (L < 0 || L > kMaxL || bwd::kNt % H != 0 || bwd::kNodeNt % H != 0) return false;
    return bwd::node_smem_floats(L, C, H, n_rbf, true) * 4 <= 227 * 1024 &&
           bwd::dw_smem_bytes(H, n_rbf) <= 227 * 1024;
}

cudaError_t run_attention_bwd(const BwdArgs& b, cudaStream_t s) {
    using namespace bwd;
    const AttnArgs& a = b.fwd;
    const int L = a.L, C = a.C, H = a.H, K = n_sh(L), N = a.n_atoms;
    const int G = (L + 1) * C + H;
    cudaError_t e;
    E2F_CUDA_TRY_E(qk_project(a.x, a.bf16, N, K, C, a.Wq, a.Wk, a.q, a.k, s));
    E2F_CUDA_TRY_E(repack_so2_f32(a.Wso2, a.bf16, L, C, a.M, a.Wt, s));
    E2F_CUDA_TRY_E(cudaMemsetAsync(b.gpos, 0, 12 * (size_t)N, s));
    E2F_CUDA_TRY_E(cudaMemsetAsync(b.gx, 0, 4 * (size_t)N * K * C, s));
    E2F_CUDA_TRY_E(cudaMemsetAsync(b.gk, 0, 4 * (size_t)N * C, s));
    E2F_CUDA_TRY_E(cudaMemsetAsync(b.gWrad, 0, 4 * (size_t)a.n_rbf * G, s));

    BwdParams P{};
    P.n_atoms = N; P.C = C; P.H = H; P.n_rbf = a.n_rbf; P.M = a.M; P.n_pairs = (int)a.n_pairs;
    P.cutoff = a.cutoff; P.box = a.box; P.pos = a.pos; P.row_ptr = a.row_ptr; P.col = a.col; P.x = a.x;
    P.W = a.Wso2; P.Wt = a.Wt; P.Wrad = a.Wrad; P.q = a.q; P.k = a.k; P.G = b.grad_out;
    P.lse = b.lse; P.beta = b.beta; P.gq = b.gq; P.gk = b.gk; P.gpos = b.gpos; P.gx = b.gx; P.gWrad = b.gWrad;
    P.gW = b.gWso2;
    P.gWpart = b.gWpart;
    P.dw_tiles = n_dw_tiles(L, C, a.M);
    P.status = b.status;

    int dev = 0, n_sm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = node_smem_floats(L, C, H, a.n_rbf, a.bf16) * 4;
    if (a.bf16) {
        P.w16 = static_cast<const __half*>(b.w16);
        P.wt16 = P.w16 + so2_total(L, C, a.M);
        count_launch();
        k_bwd_w16<__nv_bfloat16><<<592, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.Wso2), L, C, a.M,
                                                      static_cast<__half*>(b.w16),
                                                      static_cast<__half*>(b.w16) + so2_total(L, C, a.M));
        E2F_CUDA_TRY_E(cudaGetLastError());
    }
    const int grid = std::max(1, std::min(N, n_sm));
#define E2F_BWD_NODE(LL)                                                                                     \
    case LL:                                                                                                 \
        e = a.bf16 ? launch_node<LL, __nv_bfloat16>(P, smem, grid, s) : launch_node<LL, float>(P, smem, grid, s); \
        break;
    switch (L) {
        E2F_BWD_NODE(0)
        E2F_BWD_NODE(1)
        E2F_BWD_NODE(2)
        E2F_BWD_NODE(3)
        E2F_BWD_NODE(4)
        default: return cudaErrorInvalidValue;
    }
#undef E2F_BWD_NODE
    if (e != cudaSuccess) return e;
    if (b.gWq || b.gWk) {
        count_launch();
        if (a.bf16)
            k_bwd_wqk<__nv_bfloat16><<<(C * C + 255) / 256, 256, 0, s>>>(
                static_cast<const __nv_bfloat16*>(a.x), N, K, C, b.gq, b.gk, b.gWq, b.gWk);
        else
            k_bwd_wqk<float><<<(C * C + 255) / 256, 256, 0, s>>>(static_cast<const float*>(a.x), N, K, C, b.gq,
                                                                 b.gk, b.gWq, b.gWk);
        E2F_CUDA_TRY_E(cudaGetLastError());
    }
    count_launch();
    k_bwd_x0<<<(N * C + 255) / 256, 256, 0, s>>>(N, K, C, a.Wq, a.Wk, b.gq, b.gk, b.gx);
    E2F_CUDA_TRY_E(cudaGetLastError());
    if (b.gWso2 && a.n_pairs > 0 && a.bf16) {
        // operand rows per chunk of edges, then the block GEMMs over the chunk (cuBLAS)
        if (C % 8 != 0 || H > kOpsMaxH || a.n_rbf > kURbf || !b.ops) return cudaErrorInvalidValue;
        cublasHandle_t h = cublas_handle();
        if (!h) return cudaErrorNotSupported;
        if (cublas_rt().set_stream(h, s) != CUBLAS_STATUS_SUCCESS) return cudaErrorNotSupported;
        E2F_CUDA_TRY_E(cudaMemsetAsync(b.gWso2, 0, 4 * so2_total(L, C, a.M), s));
        const size_t KC = (size_t)K * C;
        __half* Xo = static_cast<__half*>(b.ops);
        __half* Yo = Xo + (size_t)std::min<int64_t>(a.n_pairs, kOpsChunk) * KC;
        for (int64_t c0 = 0; c0 < a.n_pairs; c0 += kOpsChunk) {
            const int nc = (int)std::min<int64_t>(kOpsChunk, a.n_pairs - c0);
            switch (L) {
                case 0: e = launch_ops<0>(P, (int)c0, nc, Xo, Yo, s); break;
                case 1: e = launch_ops<1>(P, (int)c0, nc, Xo, Yo, s); break;
                case 2: e = launch_ops<2>(P, (int)c0, nc, Xo, Yo, s); break;
                case 3: e = launch_ops<3>(P, (int)c0, nc, Xo, Yo, s); break;
                case 4: e = launch_ops<4>(P, (int)c0, nc, Xo, Yo, s); break;
                default: return cudaErrorInvalidValue;
            }
            if (e != cudaSuccess) return e;
            for (int mu = 0; mu <= a.M; ++mu) {
                const int nm = (L + 1 - mu) * C;
                float* dA = b.gWso2 + so2_offset(L, C, mu, 0);
                const int cp = ops_col(mu, mu, L, C), cm = ops_col(mu, -mu, L, C);
                cublasStatus_t cs;
                if (mu == 0) {
                    cs = gemm_edges(h, nm, nc, KC, Xo + cp, Yo + cp, 1.f, dA);
                } else {
                    float* dB = b.gWso2 + so2_offset(L, C, mu, 1);
                    cs = gemm_edges(h, nm, nc, KC, Xo + cp, Yo + cp, 1.f, dA);  // Y+ X+^T
                    if (cs == CUBLAS_STATUS_SUCCESS) cs = gemm_edges(h, nm, nc, KC, Xo + cm, Yo + cm, 1.f, dA);
                    if (cs == CUBLAS_STATUS_SUCCESS) cs = gemm_edges(h, nm, nc, KC, Xo + cp, Yo + cm, 1.f, dB);
                    if (cs == CUBLAS_STATUS_SUCCESS) cs = gemm_edges(h, nm, nc, KC, Xo + cm, Yo + cp, -1.f, dB);
                }
                if (cs != CUBLAS_STATUS_SUCCESS) return cudaErrorUnknown;
            }
        }
    } else if (b.gWso2 && a.n_pairs > 0) {
        const int nt = P.dw_tiles * kDwSplit;
        const size_t dsm = dw_smem_bytes(H, a.n_rbf);
#define E2F_BWD_DW(LL)                                                                                         \
    case LL:                                                                                                   \
        e = launch_dw<LL, float>(P, nt, dsm, s);                                                           \
        break;
        switch (L) {
            E2F_BWD_DW(0)
            E2F_BWD_DW(1)
            E2F_BWD_DW(2)
            E2F_BWD_DW(3)
            E2F_BWD_DW(4)
            default: return cudaErrorInvalidValue;
        }
#undef E2F_BWD_DW
        if (e != cudaSuccess) return e;
        count_launch();
        k_bwd_dw_sum<<<592, 256, 0, s>>>(b.gWpart, so2_total(L, C, a.M), b.gWso2);
        E2F_CUDA_TRY_E(cudaGetLastError());
    } else if (b.gWso2) {
        E2F_CUDA_TRY_E(cudaMemsetAsync(b.gWso2, 0, 4 * so2_total(L, C, a.M), s));
    }
    return cudaSuccess;
}

}  // namespace e2f
