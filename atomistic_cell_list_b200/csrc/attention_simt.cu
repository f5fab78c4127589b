// CUDA-core (fp32) path of the on-the-fly equivariant attention forward.
//
// One CTA per destination node i streams N(i) in tiles of TE edges
// (E2Former-V2, gist.science Technical Summary 2.2: streaming reduction with
// an online softmax whose running max, normaliser and value accumulator stay
// on chip). Per tile:
//   1 geometry: r = mic(x_j - x_i), the edge frame R, Wigner-D blocks D^l(R)
//     (Ivanic-Ruedenberg recursion), radial basis rho(d)
//   2 gates [g_v | g_a] = rho W_rad; logits a = g_a <q_i, k_j>/sqrt(d)
//   3 online softmax: new running max, rescale normaliser and accumulator
//   4 per |m| block (EAAS, 2.1: Lemma 4.1 + Eq. 13):
//       h~[l1, +-m, c] = g_v[l1,c] sum_n D^l1[+-m, n] x_j[l1, n, c]
//       o[l3, +m] = A h~+ - B h~-,  o[l3, -m] = B h~+ + A h~-
//       acc[l3, n, c] += p (D^l3[+m, n] o+ + D^l3[-m, n] o-)   (D^T o, one
//       |m| block at a time; the sum over blocks is the full rotate-back)
// No per-edge tensor leaves shared memory. All arithmetic is fp32; x and
// W_so2 may be stored in bf16. This path serves fp32 features (where bf16
// tensor cores cannot meet the fp32 tolerance) and is the reference-quality
// GPU implementation.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "attention.cuh"
#include "common.cuh"

namespace e2f {

// q = W_q x[l=0], k = W_k x[l=0]  (Eq. 6: invariant scalar projections)
template <typename T>
__global__ void k_qk_project(const T* __restrict__ x, int n_atoms, int K, int C, const float* __restrict__ Wq,
                             const float* __restrict__ Wk, float* q, float* k) {
    extern __shared__ float xs[];
    const int i = blockIdx.x;
    for (int c = threadIdx.x; c < C; c += blockDim.x) xs[c] = load_feat(x, (size_t)i * K * C + c);
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        float sq = 0.f, sk = 0.f;
        for (int c2 = 0; c2 < C; ++c2) {
            sq = fmaf(Wq[(size_t)c * C + c2], xs[c2], sq);
            sk = fmaf(Wk[(size_t)c * C + c2], xs[c2], sk);
        }
        q[(size_t)i * C + c] = sq;
        k[(size_t)i * C + c] = sk;
    }
}

// Packed SO(2) blocks (row-major [(l3,c_out),(l1,c_in)]) -> fp32, each block
// transposed so that consecutive output rows are consecutive in memory.
template <typename T>
__global__ void k_repack_so2_f32(const T* __restrict__ w, int L, int C, int M, float* out) {
    const size_t total = so2_total(L, C, M);
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        size_t off = 0;
        int n = (L + 1) * C;
        int blk = 0;
        while (e >= off + (size_t)n * n) {
            off += (size_t)n * n;
            ++blk;
            const int m = (blk + 1) / 2;
            n = (L + 1 - m) * C;
        }
        const size_t loc = e - off;
        const int r = (int)(loc / n), kk = (int)(loc % n);
        out[off + (size_t)kk * n + r] = load_feat(w, e);
    }
}

struct SimtParams {
    int n_atoms, C, H, n_rbf;
    int M;  // SO(2) maps for |m| <= M
    float cutoff;
    Box box;
    const float* pos;
    const int32_t* row_ptr;
    const int32_t* col;
    const void* x;
    const float* q;
    const float* k;
    const float* Wrad;
    const float* Wt;  // repacked SO(2) weights (see k_repack_so2_f32)
    float* out;
    int te;           // edges per tile (multiple of 4)
};

template <int L, typename T>
__global__ void __launch_bounds__(256) k_attn_simt(SimtParams P) {
    constexpr int K = n_sh(L);
    constexpr int WS = wig_size(L);
    const int C = P.C, H = P.H, dh = C / H, te = P.te, nr = P.n_rbf;
    const int G = (L + 1) * C + H;                           // gate columns
    const int KH = (L >= 1) ? max((L + 1) * C, 2 * L * C) : C;  // largest block input
    const T* __restrict__ x = static_cast<const T*>(P.x);

    extern __shared__ float sm[];
    float* acc = sm;                       // [K][C]
    float* Dm = acc + K * C;               // [te][WS]
    float* rho = Dm + te * WS;             // [te][nr]
    float* g = rho + te * nr;              // [te][G]
    float* hs = g + te * G;                // [KH][te]
    float* pw = hs + KH * te;              // [te][H]  softmax weights of the tile
    float* run_m = pw + te * H;            // [H]
    float* run_s = run_m + H;              // [H]
    float* scl = run_s + H;                // [H]
    int* jn = reinterpret_cast<int*>(scl + H);  // [te]

    const int i = blockIdx.x;
    const int e_begin = P.row_ptr[i], e_end = P.row_ptr[i + 1];
    const int tid = threadIdx.x, nt = blockDim.x;

    for (int t = tid; t < K * C; t += nt) acc[t] = 0.f;
    for (int h = tid; h < H; h += nt) { run_m[h] = -INFINITY; run_s[h] = 0.f; }
    __syncthreads();

    const float inv_sqrt_dh = rsqrtf((float)dh);
    for (int e0 = e_begin; e0 < e_end; e0 += te) {
        const int ne = min(te, e_end - e0);
        // 1 geometry, frame, Wigner blocks, radial basis (one thread per edge)
        if (tid < te) {
            float* D = Dm + tid * WS;
            if (tid < ne) {
                const int j = P.col[e0 + tid];
                jn[tid] = j;
                float3 r = edge_vec(P.pos, i, j, P.box);
                const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
                float R[3][3];
                edge_frame(r.x / d, r.y / d, r.z / d, R);
                wigner_blocks<L>(R, D);
                for (int kb = 0; kb < nr; ++kb) rho[tid * nr + kb] = rbf(d, kb, P.cutoff, nr);
            } else {
                jn[tid] = i;
                for (int a = 0; a < WS; ++a) D[a] = 0.f;
                for (int kb = 0; kb < nr; ++kb) rho[tid * nr + kb] = 0.f;
            }
        }
        __syncthreads();
        // 2 gates
        for (int t = tid; t < te * G; t += nt) {
            const int e = t / G, c = t % G;
            float s = 0.f;
            for (int kb = 0; kb < nr; ++kb) s = fmaf(rho[e * nr + kb], P.Wrad[(size_t)kb * G + c], s);
            g[t] = s;
        }
        __syncthreads();
        // 3 logits and online softmax (running max m, normaliser s)
        for (int t = tid; t < te * H; t += nt) {
            const int e = t / H, h = t % H;
            float a = -INFINITY;
            if (e < ne) {
                const float* qi = P.q + (size_t)i * C + h * dh;
                const float* kj = P.k + (size_t)jn[e] * C + h * dh;
                float dot = 0.f;
                for (int c = 0; c < dh; ++c) dot = fmaf(qi[c], kj[c], dot);
                a = g[e * G + (L + 1) * C + h] * dot * inv_sqrt_dh;
            }
            pw[t] = a;
        }
        __syncthreads();
        for (int h = tid; h < H; h += nt) {
            float mt = -INFINITY;
            for (int e = 0; e < ne; ++e) mt = fmaxf(mt, pw[e * H + h]);
            const float mn = fmaxf(run_m[h], mt);
            const float sc = expf(run_m[h] - mn);  // 0 on the first tile
            float s = run_s[h] * sc;
            for (int e = 0; e < te; ++e) {
                const float p = (e < ne) ? expf(pw[e * H + h] - mn) : 0.f;
                pw[e * H + h] = p;
                s += p;
            }
            run_m[h] = mn;
            run_s[h] = s;
            scl[h] = sc;
        }
        __syncthreads();
        if (e0 != e_begin)
            for (int t = tid; t < K * C; t += nt) acc[t] *= scl[(t % C) / dh];
        __syncthreads();

        // 4 per |m| block
#pragma unroll 1
        for (int m = 0; m <= P.M; ++m) {  // |m| > M: no message (truncated layer)
            const int nm = (L + 1 - m) * C;         // rows (and columns) of A(m)
            // 4a rotated, gated block input: hs[(s, l1-m, c)][e]
            for (int t = tid; t < te * nm; t += nt) {
                const int e = t / nm, r = t % nm;
                const int l1 = m + r / C, c = r % C;
                float vp = 0.f, vm = 0.f;
                if (e < ne) {
                    const float* D = Dm + e * WS + wig_off(l1);
                    const int w = 2 * l1 + 1;
                    const size_t xb = ((size_t)jn[e] * K + l1 * l1) * C + c;
                    for (int n = 0; n < w; ++n) {
                        const float xv = load_feat(x, xb + (size_t)n * C);
                        vp = fmaf(D[(l1 + m) * w + n], xv, vp);
                        vm = fmaf(D[(l1 - m) * w + n], xv, vm);
                    }
                    const float gv = g[e * G + l1 * C + c];
                    vp *= gv;
                    vm *= gv;
                }
                hs[(size_t)r * te + e] = vp;
                if (m > 0) hs[(size_t)(nm + r) * te + e] = vm;
            }
            __syncthreads();
            // 4b SO(2) block product and partial rotate-back into acc
            const float* At = P.Wt + so2_offset(L, C, m, 0);
            const float* Bt = (m > 0) ? P.Wt + so2_offset(L, C, m, 1) : nullptr;
            for (int r = tid; r < nm; r += nt) {
                const int l3 = m + r / C, c = r % C, h = c / dh;
                float op[16], om[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) { op[e] = 0.f; om[e] = 0.f; }
                for (int kk = 0; kk < nm; ++kk) {
                    const float a = At[(size_t)kk * nm + r];
                    const float4* hp = reinterpret_cast<const float4*>(hs + (size_t)kk * te);
                    if (m == 0) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            if (q4 * 4 < te) {
                                float4 v = hp[q4];
                                op[q4 * 4 + 0] = fmaf(a, v.x, op[q4 * 4 + 0]);
                                op[q4 * 4 + 1] = fmaf(a, v.y, op[q4 * 4 + 1]);
                                op[q4 * 4 + 2] = fmaf(a, v.z, op[q4 * 4 + 2]);
                                op[q4 * 4 + 3] = fmaf(a, v.w, op[q4 * 4 + 3]);
                            }
                        }
                    } else {
                        const float b = Bt[(size_t)kk * nm + r];
                        const float4* hmn = reinterpret_cast<const float4*>(hs + (size_t)(nm + kk) * te);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            if (q4 * 4 < te) {
                                float4 u = hp[q4], v = hmn[q4];
                                op[q4 * 4 + 0] = fmaf(a, u.x, fmaf(-b, v.x, op[q4 * 4 + 0]));
                                op[q4 * 4 + 1] = fmaf(a, u.y, fmaf(-b, v.y, op[q4 * 4 + 1]));
                                op[q4 * 4 + 2] = fmaf(a, u.z, fmaf(-b, v.z, op[q4 * 4 + 2]));
                                op[q4 * 4 + 3] = fmaf(a, u.w, fmaf(-b, v.w, op[q4 * 4 + 3]));
                                om[q4 * 4 + 0] = fmaf(b, u.x, fmaf(a, v.x, om[q4 * 4 + 0]));
                                om[q4 * 4 + 1] = fmaf(b, u.y, fmaf(a, v.y, om[q4 * 4 + 1]));
                                om[q4 * 4 + 2] = fmaf(b, u.z, fmaf(a, v.z, om[q4 * 4 + 2]));
                                om[q4 * 4 + 3] = fmaf(b, u.w, fmaf(a, v.w, om[q4 * 4 + 3]));
                            }
                        }
                    }
                }
                const int w3 = 2 * l3 + 1;
                float* ac = acc + (size_t)(l3 * l3) * C + c;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    if (e < ne) {
                        const float p = pw[e * H + h];
                        const float* D = Dm + e * WS + wig_off(l3);
                        const float vp = p * op[e], vm = p * om[e];
                        for (int n = 0; n < w3; ++n) {
                            float v = D[(l3 + m) * w3 + n] * vp;
                            if (m > 0) v = fmaf(D[(l3 - m) * w3 + n], vm, v);
                            ac[(size_t)n * C] += v;
                        }
                    }
                }
            }
            __syncthreads();
        }
    }
    // finalize: divide by the normaliser; isolated nodes give 0
    for (int t = tid; t < K * C; t += nt) {
        const int h = (t % C) / dh;
        P.out[(size_t)i * K * C + t] = (e_end > e_begin) ? acc[t] / run_s[h] : 0.f;
    }
}

size_t simt_smem_bytes(int L, int C, int H, int n_rbf, int te) {
    const int K = n_sh(L), WS = wig_size(L), G = (L + 1) * C + H;
    const int KH = (L >= 1) ? std::max((L + 1) * C, 2 * L * C) : C;
    size_t f = (size_t)K * C + (size_t)te * WS + (size_t)te * n_rbf + (size_t)te * G + (size_t)KH * te +
               (size_t)te * H + 3 * (size_t)H;
    return f * 4 + (size_t)te * 4 + 16;
}

template <int L, typename T>
static cudaError_t launch_simt_t(const SimtParams& P, size_t smem, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_simt<L, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    k_attn_simt<L, T><<<P.n_atoms, 256, smem, s>>>(P);
    return cudaGetLastError();
}

cudaError_t run_attention_simt(const AttnArgs& a, cudaStream_t s) {
    const int C = a.C, K = n_sh(a.L);
    // Q/K projections and weight repack
    if (a.bf16) {
        count_launch();
        k_qk_project<__nv_bfloat16><<<a.n_atoms, 128, C * 4, s>>>(static_cast<const __nv_bfloat16*>(a.x), a.n_atoms,
                                                                  K, C, a.Wq, a.Wk, a.q, a.k);
        count_launch();
        k_repack_so2_f32<__nv_bfloat16><<<1184, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.Wso2), a.L, C, a.M,
                                                             a.Wt);
    } else {
        count_launch();
        k_qk_project<float><<<a.n_atoms, 128, C * 4, s>>>(static_cast<const float*>(a.x), a.n_atoms, K, C, a.Wq,
                                                          a.Wk, a.q, a.k);
        count_launch();
        k_repack_so2_f32<float><<<1184, 256, 0, s>>>(static_cast<const float*>(a.Wso2), a.L, C, a.M, a.Wt);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    SimtParams P;
    P.n_atoms = a.n_atoms; P.C = C; P.H = a.H; P.n_rbf = a.n_rbf; P.M = a.M; P.cutoff = a.cutoff; P.box = a.box;
    P.pos = a.pos; P.row_ptr = a.row_ptr; P.col = a.col; P.x = a.x; P.q = a.q; P.k = a.k;
    P.Wrad = a.Wrad; P.Wt = a.Wt; P.out = a.out;
    int te = 16;
    while (te > 4 && simt_smem_bytes(a.L, C, a.H, a.n_rbf, te) > 220 * 1024) te /= 2;
    P.te = te;
    const size_t smem = simt_smem_bytes(a.L, C, a.H, a.n_rbf, te);
#define E2F_SIMT_CASE(LL)                                                                   \
    case LL:                                                                                \
        return a.bf16 ? launch_simt_t<LL, __nv_bfloat16>(P, smem, s) : launch_simt_t<LL, float>(P, smem, s);
    switch (a.L) {
        E2F_SIMT_CASE(0)
        E2F_SIMT_CASE(1)
        E2F_SIMT_CASE(2)
        E2F_SIMT_CASE(3)
        E2F_SIMT_CASE(4)
        default: return cudaErrorInvalidValue;
    }
#undef E2F_SIMT_CASE
}

cudaError_t qk_project(const void* x, bool bf16, int n_atoms, int K, int C, const float* Wq, const float* Wk,
                       float* q, float* k, cudaStream_t s) {
    count_launch();
    if (bf16)
        k_qk_project<__nv_bfloat16><<<n_atoms, 128, C * 4, s>>>(static_cast<const __nv_bfloat16*>(x), n_atoms, K, C,
                                                                Wq, Wk, q, k);
    else
        k_qk_project<float><<<n_atoms, 128, C * 4, s>>>(static_cast<const float*>(x), n_atoms, K, C, Wq, Wk, q, k);
    return cudaGetLastError();
}

cudaError_t repack_so2_f32(const void* w, bool bf16, int L, int C, int M, float* out, cudaStream_t s) {
    count_launch();
    if (bf16)
        k_repack_so2_f32<__nv_bfloat16><<<1184, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), L, C, M, out);
    else
        k_repack_so2_f32<float><<<1184, 256, 0, s>>>(static_cast<const float*>(w), L, C, M, out);
    return cudaGetLastError();
}

// Wigner blocks for a batch of directions (exposed for testing the rotation)
template <int L>
__global__ void k_edge_wigner(const float* r, int64_t n, float* out, float* frames) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n) return;
    const float x = r[3 * e], y = r[3 * e + 1], z = r[3 * e + 2];
    const float d = sqrtf(x * x + y * y + z * z);
    float R[3][3];
    edge_frame(x / d, y / d, z / d, R);
    float D[wig_size(L)];
    wigner_blocks<L>(R, D);
    for (int a = 0; a < wig_size(L); ++a) out[e * wig_size(L) + a] = D[a];
    if (frames)
        for (int a = 0; a < 9; ++a) frames[e * 9 + a] = R[a / 3][a % 3];
}

cudaError_t run_edge_wigner(const float* r, int64_t n, int L, float* out, float* frames, cudaStream_t s) {
    const unsigned nb = (unsigned)((n + 127) / 128);
    count_launch();
    switch (L) {
        case 0: k_edge_wigner<0><<<nb, 128, 0, s>>>(r, n, out, frames); break;
        case 1: k_edge_wigner<1><<<nb, 128, 0, s>>>(r, n, out, frames); break;
        case 2: k_edge_wigner<2><<<nb, 128, 0, s>>>(r, n, out, frames); break;
        case 3: k_edge_wigner<3><<<nb, 128, 0, s>>>(r, n, out, frames); break;
        case 4: k_edge_wigner<4><<<nb, 128, 0, s>>>(r, n, out, frames); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace e2f
