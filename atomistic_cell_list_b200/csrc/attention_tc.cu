// Tensor-core (tcgen05) path of the on-the-fly equivariant attention forward
// for bf16 features (E2Former-V2, gist.science Technical Summary 2.1-2.2).
//
// Work split. A persistent CTA per SM owns a contiguous range of destination
// nodes (balanced by edge count) and walks its edges in tiles of 128 (CSR
// order). The SO(2) maps (EAAS, Eq. 13) are one GEMM per |m| block,
// written transposed so that the 128 TMEM lanes are output features and the
// 128 columns are the tile's edges:
//
//   o+[f, e] = sum_k A(m)[f, k] h+[e, k] - B(m)[f, k] h-[e, k]
//   o-[f, e] = sum_k B(m)[f, k] h+[e, k] + A(m)[f, k] h-[e, k]
//
// A and B are read by TMA from fp16 copies of the packed weights (the A
// operand, K-major); h = the tile's rotated, gated neighbour features (the
// B operand, K-major). One A/B weight tile serves two MMAs (the -B product
// uses the instruction's negate bit). A group = up to two accumulators (o+
// and o- of the same features, or two feature blocks of m = 0) = 256 TMEM
// columns; two groups in flight let the epilogue drain one while the MMA
// fills the other.
//
// Warp roles (512 threads, 128 registers each):
//   0-3, 8-11  epilogue: tcgen05.ld 16x256b fragments of the accumulators;
//              rotate-back p * D^l3(R)^T restricted to the group's |m| rows
//              on mma.sync, summed over each node's edges, added to
//              out[node] (one owner thread per element: fixed order)
//   4-7        producer: per edge the node, frame, Wigner blocks (fp16 pairs,
//              shared and global copies); per (edge, head) the softmax weight
//              p = exp(a - lse) (statistics from an O(N) pre-pass); per
//              (edge, 8 channels) the gathered, gated, rotated features,
//              written once per tile to a per-CTA global scratch row for TMA
//   12         TMA loads of weight and feature tiles into a 3-stage ring
//   13         tcgen05.mma issue (one thread), commits to the ring and TMEM
//              barriers
//   14-15      value gates rho(d) W_rad of a tile (mma.sync), up to two tiles
//              ahead of the producer, into a double-buffered global scratch
// Every mbarrier wait is bounded by the global timer; on expiry the kernel
// records E2F_ERR_TIMEOUT, drains what it issued and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <algorithm>

#include "attention.cuh"
#include "attention_tc.cuh"
#include "cell_grid.cuh"
#include "common.cuh"
#include "tcgen05.cuh"

namespace e2f {
namespace tc {

// K-major operand tile of 128 rows x 32 bf16 (64-byte rows), 64-byte swizzle:
// 8-row core groups 512 bytes apart; the second K=16 step starts 32 bytes in.
__device__ __forceinline__ uint64_t sdesc_sw64(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;               // leading byte offset (unused when swizzled)
    d |= (uint64_t)(512u >> 4) << 32;      // stride byte offset: 8 rows x 64 B
    d |= (uint64_t)1u << 46;               // descriptor version (sm_100)
    d |= (uint64_t)4u << 61;               // SWIZZLE_64B
    return d;
}

// kind::f16 instruction descriptor: D fp32, A and B fp16 (format 0), both
// K-major, M = 128, N = 128, optional negation of A.
__host__ __device__ constexpr uint32_t idesc_f16(bool neg_a) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((neg_a ? 1u : 0u) << 13) | ((128u >> 3) << 17) |
           ((128u >> 4) << 24);
}

// ----------------------------------------------------------------------------
// pre-passes
// ----------------------------------------------------------------------------
// Softmax statistics per node and head, lse = m + log(sum exp(a - m)), by an
// online max/sum over the node's edges. One warp per node; lane = (edge slot
// es, head h) with 32 / H edge slots, so a head's q and logit-gate column
// stay in registers and the key row of an edge is read as float4 by its H
// lanes. The logit is evaluated in the same order as in the main kernel.
__global__ void __launch_bounds__(256) k_softmax_stats(StatsParams P) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= P.n_atoms) return;
    const int i = warp;
    const int H = P.H, C = P.C, dh = C / H, G = P.G, Gv = G - H;
    const int h = lane % H, es = lane / H, EP = 32 / H;
    const float inv = rsqrtf((float)dh);
    float wcol[kTcMaxRbf];
#pragma unroll
    for (int kb = 0; kb < kTcMaxRbf; ++kb) wcol[kb] = kb < P.n_rbf ? P.Wrad[(size_t)kb * G + Gv + h] : 0.f;
    const float4* q4 = reinterpret_cast<const float4*>(P.q + (size_t)i * C + h * dh);
    const int d4 = dh / 4;
    float m = -INFINITY, s = 0.f;
    const int e0 = P.row_ptr[i], e1 = P.row_ptr[i + 1];
    for (int e = e0 + es; e < e1; e += EP) {
        const int j = P.col[e];
        const float3 r = edge_vec(P.pos, i, j, P.box);
        const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
        float rr[kTcMaxRbf];
        rbf_all<kTcMaxRbf>(d, P.cutoff, P.n_rbf, rr);
        float ga = 0.f;
#pragma unroll
        for (int kb = 0; kb < kTcMaxRbf; ++kb) ga = fmaf(rr[kb], wcol[kb], ga);
        const float4* k4 = reinterpret_cast<const float4*>(P.k + (size_t)j * C + h * dh);
        float dot = 0.f;
        for (int c4 = 0; c4 < d4; ++c4) {
            const float4 qa = __ldg(q4 + c4), kv = __ldg(k4 + c4);
            dot = fmaf(qa.x, kv.x, dot);
            dot = fmaf(qa.y, kv.y, dot);
            dot = fmaf(qa.z, kv.z, dot);
            dot = fmaf(qa.w, kv.w, dot);
        }
        const float a = ga * dot * inv;
        const float mn = fmaxf(m, a);
        s = s * expf(m - mn) + expf(a - mn);
        m = mn;
    }
    // combine the edge slots of each head
    for (int o = H; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o), so = __shfl_xor_sync(0xffffffffu, s, o);
        const float mn = fmaxf(m, mo);
        const float sa = (m == -INFINITY) ? 0.f : s * expf(m - mn);
        const float sb = (mo == -INFINITY) ? 0.f : so * expf(mo - mn);
        m = mn;
        s = sa + sb;
    }
    if (es == 0) P.lse[(size_t)i * H + h] = (e1 > e0) ? m + logf(s) : 0.f;
}

// The same statistics with the neighbours enumerated from the cell lists
// (fused traversal): one warp per node slot in cell order. The warp collects
// the node's neighbours in shared memory, kStatsCap at a time (a denser node
// enumerates again for the next window), then evaluates them with the lane
// layout and per-edge arithmetic of k_softmax_stats.
constexpr int kStatsCap = 256;
__global__ void __launch_bounds__(256) k_softmax_stats_cells(StatsParams P, CellView cv) {
    __shared__ int jbuf[8][kStatsCap];
    const int s = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (s >= P.n_atoms) return;
    int* jb = jbuf[threadIdx.x >> 5];
    const int H = P.H, C = P.C, dh = C / H, G = P.G, Gv = G - H;
    const int h = lane % H, es = lane / H, EP = 32 / H;
    const float inv = rsqrtf((float)dh);
    float wcol[kTcMaxRbf];
#pragma unroll
    for (int kb = 0; kb < kTcMaxRbf; ++kb) wcol[kb] = kb < P.n_rbf ? P.Wrad[(size_t)kb * G + Gv + h] : 0.f;
    const int i = cv.sidx[s];
    const float4 me = cv.spos[s];
    const float4* q4 = reinterpret_cast<const float4*>(P.q + (size_t)i * C + h * dh);
    const int d4 = dh / 4;
    float m = -INFINITY, sum = 0.f;
    int cnt = 0;
    for (int w0 = 0;; w0 += kStatsCap) {
        cnt = warp_neighbors(
            cv, me, i,
            [&](int k, int j) {
                if (k >= w0 && k < w0 + kStatsCap) jb[k - w0] = j;
            },
            0, s);
        __syncwarp();
        const int n_here = min(cnt - w0, kStatsCap);
        for (int k = es; k < n_here; k += EP) {
            const int j = jb[k];
            const float3 r = edge_vec(P.pos, i, j, P.box);
            const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
            float rr[kTcMaxRbf];
            rbf_all<kTcMaxRbf>(d, P.cutoff, P.n_rbf, rr);
            float ga = 0.f;
#pragma unroll
            for (int kb = 0; kb < kTcMaxRbf; ++kb) ga = fmaf(rr[kb], wcol[kb], ga);
            const float4* k4 = reinterpret_cast<const float4*>(P.k + (size_t)j * C + h * dh);
            float dot = 0.f;
            for (int c4 = 0; c4 < d4; ++c4) {
                const float4 qa = __ldg(q4 + c4), kv = __ldg(k4 + c4);
                dot = fmaf(qa.x, kv.x, dot);
                dot = fmaf(qa.y, kv.y, dot);
                dot = fmaf(qa.z, kv.z, dot);
                dot = fmaf(qa.w, kv.w, dot);
            }
            const float a = ga * dot * inv;
            const float mn = fmaxf(m, a);
            sum = sum * expf(m - mn) + expf(a - mn);
            m = mn;
        }
        __syncwarp();
        if (cnt <= w0 + kStatsCap) break;
    }
    for (int o = H; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o), so = __shfl_xor_sync(0xffffffffu, sum, o);
        const float mn = fmaxf(m, mo);
        const float sa = (m == -INFINITY) ? 0.f : sum * expf(m - mn);
        const float sb = (mo == -INFINITY) ? 0.f : so * expf(mo - mn);
        m = mn;
        sum = sa + sb;
    }
    if (es == 0) P.lse[(size_t)i * H + h] = (cnt > 0) ? m + logf(sum) : 0.f;
}

__global__ void k_flags_to_status(const int* flags, int* status) {
    const int f = *flags;
    if (f & kFlagNonFinite) atomicExch(status, (int)E2F_ERR_NONFINITE);
    else if (f & kFlagStale) atomicExch(status, (int)E2F_ERR_STALE);
}

// Node range per CTA: part[k] = first node whose edges start at or after
// k * E / n_ctas (so a node never spans two CTAs).
__global__ void k_partition(const int32_t* row_ptr, int n_atoms, int n_ctas, int32_t* part) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k > n_ctas) return;
    if (k == n_ctas) { part[k] = n_atoms; return; }
    const long long E = row_ptr[n_atoms];
    const long long target = E * k / n_ctas;
    int lo = 0, hi = n_atoms;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (row_ptr[mid] < target) lo = mid + 1; else hi = mid;
    }
    part[k] = lo;
}

// Q/K projection (Eq. 6): q = W_q x[l=0], k = W_k x[l=0], as one [N x C] x [C x 2C]
// product on the FP32 pipe. A CTA computes 64 nodes x 64 outputs (outputs
// o < C are q, the rest k); K = C runs in chunks of 32 through shared memory:
// the features node-major (row stride 33: conflict-free stores of coalesced
// reads), the weights k-major (a thread reads its 4 outputs of a k step as one
// float4). Each of the 256 threads accumulates a 4 x 4 block.
constexpr int kQkM = 64, kQkN = 64, kQkK = 32;
__global__ void __launch_bounds__(256) k_qk_tiled(const __nv_bfloat16* __restrict__ x, int n_atoms, int K, int C,
                                                   const float* __restrict__ Wq, const float* __restrict__ Wk,
                                                   float* q, float* k) {
    __shared__ float xs[kQkM][kQkK + 1];
    __shared__ __align__(16) float ws[kQkK][kQkN];
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int n0 = blockIdx.x * kQkM, o0 = blockIdx.y * kQkN;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    for (int c0 = 0; c0 < C; c0 += kQkK) {
        __syncthreads();
        for (int t = tid; t < kQkM * kQkK; t += 256) {
            const int a = t / kQkK, kk = t % kQkK;  // consecutive threads: consecutive channels of a node
            const int n = n0 + a;
            xs[a][kk] = n < n_atoms ? __bfloat162float(x[(size_t)n * K * C + c0 + kk]) : 0.f;
        }
        for (int t = tid; t < kQkN * kQkK; t += 256) {
            const int o = t % kQkN, kk = t / kQkN;  // consecutive threads: consecutive outputs
            const int og = o0 + o;
            const float* W = og < C ? Wq + (size_t)og * C : Wk + (size_t)(og - C) * C;
            ws[kk][o] = og < 2 * C ? W[c0 + kk] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kQkK; ++kk) {
            const float4 wb = *reinterpret_cast<const float4*>(&ws[kk][4 * tx]);
            const float wv[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float xv = xs[4 * ty + a][kk];
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(xv, wv[b], acc[a][b]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int n = n0 + 4 * ty + a;
        if (n >= n_atoms) continue;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int og = o0 + 4 * tx + b;
            if (og < C) q[(size_t)n * C + og] = acc[a][b];
            else if (og < 2 * C) k[(size_t)n * C + og - C] = acc[a][b];
        }
    }
}

// ----------------------------------------------------------------------------
// fp16 operand preparation. The tensor cores take fp16 (3 more mantissa bits
// than bf16). Features are scaled by an exact power of two s so that
// |s x| <= 1; the gate bound n_rbf * max|W_rad| then keeps every rotated,
// gated value far inside the fp16 range (checked). The output is linear in x
// through the value path, so multiplying the softmax weights by 1/s restores
// it exactly.
// ----------------------------------------------------------------------------
__global__ void k_amax(const __nv_bfloat16* __restrict__ x, size_t n, const float* __restrict__ w, size_t nw,
                       unsigned* amax) {
    float mx = 0.f, mw = 0.f;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n / 8; i += stride) {
        const uint4 u = reinterpret_cast<const uint4*>(x)[i];
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(h[q]);
            mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nw; i += stride) mw = fmaxf(mw, fabsf(w[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, o));
    }
    if ((threadIdx.x & 31) == 0) {  // non-negative floats order like their bit patterns
        atomicMax(amax, __float_as_uint(mx));
        atomicMax(amax + 1, __float_as_uint(mw));
    }
}

__global__ void k_make_scale(const unsigned* amax, int n_rbf, float* scale, int* status) {
    const float mx = __uint_as_float(amax[0]), mw = __uint_as_float(amax[1]);
    int e = 0;
    if (mx > 0.f && isfinite(mx)) e = ilogbf(mx) + 1;  // s x in (-1, 1)
    e = max(-60, min(60, e));
    scale[0] = ldexpf(1.f, -e);
    scale[1] = ldexpf(1.f, e);
    // |rotated gated value| <= sqrt(2l+1) |s x| |g| <= 3 n_rbf max|W_rad|
    if (!(isfinite(mx) && isfinite(mw)) || 3.f * n_rbf * mw > 16384.f) atomicExch(status, (int)E2F_ERR_UNSUPPORTED);
}

__global__ void k_x_to_f16(const __nv_bfloat16* __restrict__ x, size_t n, const float* __restrict__ scale,
                           __half* __restrict__ out) {
    const float s = scale[0];
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n / 8; i += stride) {
        const uint4 u = reinterpret_cast<const uint4*>(x)[i];
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
        uint4 v;
        __half2* o = reinterpret_cast<__half2*>(&v);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(h[q]);
            o[q] = __floats2half2_rn(f.x * s, f.y * s);
        }
        reinterpret_cast<uint4*>(out)[i] = v;
    }
}

__global__ void k_w_to_f16(const __nv_bfloat16* __restrict__ w, size_t n, __half* __restrict__ out) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        out[i] = __float2half_rn(__bfloat162float(w[i]));
}

// value-gate weights transposed to [(L+1)C][16] fp16 (radial index innermost)
__global__ void k_wrad_t(const float* __restrict__ Wrad, int n_rbf, int G, int Gv, __half* __restrict__ whT) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= Gv * kTcMaxRbf) return;
    const int n = t / kTcMaxRbf, k = t % kTcMaxRbf;
    whT[t] = __float2half_rn(k < n_rbf ? Wrad[(size_t)k * G + n] : 0.f);
}

__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// ----------------------------------------------------------------------------
// main kernel
// ----------------------------------------------------------------------------
constexpr int kTileE = 128;
constexpr int kKS = 32;                       // K per ring stage
constexpr int kNS = 3;                        // ring stages
constexpr int kSlot = kTileE * kKS * 2;       // 8 KB per operand tile
constexpr int kStage = 4 * kSlot;
constexpr int kThreads = 512;
// Warp roles (16 warps, 65536 / 512 = 128 registers per thread):
//   0-3, 8-11  epilogue (warp w: TMEM lane quadrant w % 4, lane half w / 8)
//   4-7        producer
//   12         TMA, 13 MMA, 14-15 idle
constexpr int kEpiThreads = 256;
constexpr int kChunk = 16;                    // epilogue: edges per TMEM load

// Wigner blocks of an edge in "pair" form: for each degree l and each
// |m| = mu <= l the 2l+1 pairs (D^l[+mu][n], D^l[-mu][n]) as fp16x2, padded
// to npair(l) = a multiple of 4 pairs so that a block is read with 16-byte
// loads. A pair rotates into both x~[+mu] and x~[-mu] (producer) and rotates
// o+ and o- back (epilogue). Block (l, mu) of an edge starts at pair dpo(l, mu).
__host__ __device__ constexpr int npair(int l) { return (2 * l + 4) & ~3; }
__host__ __device__ constexpr int dpo(int l, int mu) {
    int o = 0;
    for (int k = 0; k < l; ++k) o += (k + 1) * npair(k);
    return o + mu * npair(l);
}
__host__ __device__ constexpr int dptotal(int L) { return dpo(L + 1, 0); }  // 128 at L = 4
// shared copy (producer): [edge][dptotal + 4] pairs; the 4 spare pairs move
// consecutive edges 4 banks apart
__host__ __device__ constexpr int dph_stride(int L) { return dptotal(L) + 4; }
// global copy (epilogue), per tile buffer, block-major: block (l, mu) holds
// 128 edges x npair(l) pairs, so a group's slice is one bulk copy
__host__ __device__ constexpr size_t dglob_pairs() { return (size_t)kTileE * dptotal(kMaxL); }
__host__ __device__ constexpr size_t dglob_block(int l, int mu) { return (size_t)kTileE * dpo(l, mu); }
static_assert(npair(0) == 4 && npair(1) == 4 && npair(2) == 8 && npair(3) == 8 && npair(4) == 12, "pairs");
static_assert(dptotal(4) == 128, "pair layout");

// Degrees of the rows of a group: its 128-row blocks (one, or two for m = 0)
// start at rows row0 (and row0b) of the |m| section, whose rows are (l3, c)
// with l3 from |m| (m > 0) or 0 upwards; a block holds 128 / C degrees when
// C = 64. The range [lo, hi] is contiguous and clipped to L (rows past the
// section are zero-filled padding).
__host__ __device__ inline void group_l3_range(const TcGroup& g, int L, int C, int& lo, int& hi) {
    const int base = g.mu > 0 ? g.mu : 0;
    const int last = (g.mu == 0 && g.row0b >= 0) ? g.row0b : g.row0;
    lo = base + g.row0 / C;
    hi = min(L, base + (last + 127) / C);
}
__host__ __device__ inline int pairs_in(int lo, int hi) {
    int n = 0;
    for (int l = lo; l <= hi; ++l) n += npair(l);
    return n;
}

// Bytes of Wigner pairs one group's epilogue stages: npair(l3) pairs of 4
// bytes per edge for each degree l3 of the group's rows (largest over the
// groups of a layer).
__host__ __device__ inline size_t stage_bytes(int L, int C) {
    int mx = 0;
    for (int mu = 0; mu <= L; ++mu) {
        const int nm = (L + 1 - mu) * C, step = mu > 0 ? 128 : 256;
        for (int r0 = 0; r0 < nm; r0 += step) {
            TcGroup g{};
            g.mu = mu; g.row0 = r0; g.row0b = (mu == 0 && r0 + 128 < nm) ? r0 + 128 : -1;
            int lo, hi;
            group_l3_range(g, L, C, lo, hi);
            mx = max(mx, pairs_in(lo, hi));
        }
    }
    return (size_t)kTileE * 4 * mx;
}

// Shared memory layout (bytes), shared by host (size) and device (offsets).
struct SmemLayout {
    size_t ring, dstage, dstride, dph, pch, nid, jn, segm, rpw, rho, rrs, wga, bars, misc, dsub, total;
    __host__ __device__ SmemLayout(int L, int C, int H, int n_rbf) {
        size_t o = 0;
        ring = o;   o += (size_t)kNS * kStage;
        dstride = (stage_bytes(L, C) + 127) & ~size_t(127);
        dstage = o; o += 2 * dstride;
        dph = o;    o += (size_t)kTileE * dph_stride(L) * 4;
        pch = o;    o += 2ull * kTileE * (C / 8) * 4;
        nid = o;    o += 2ull * kTileE * 4;
        jn = o;     o += 2ull * kTileE * 4;
        segm = o;   o += 2ull * (kTileE / kChunk) * 4;
        rpw = o;    o += (size_t)kTileE * 4;
        rho = o;    o += (size_t)kTileE * kTcMaxRbf * 2;
        rrs = o;    o += (size_t)kTileE * kTcMaxRbf * 4;
        wga = o;    o += (size_t)kTcMaxRbf * kMaxHeads * 4;
        o = (o + 7) & ~size_t(7);
        bars = o;   o += (2 * kNS + 17) * 8;
        misc = o;   o += 64 + 4 * kTileE * 4;  // TMEM base, abort flag, last slot; gate (i, j) lists
        dsub = o;   o += 16 * 8;
        total = o;
    }
};

__device__ __forceinline__ int kpos(int l1, int m, int L, int C) {
    // column of (l1, m) in a scratch row: m = 0 block, then (+m, -m) halves per |m|
    const int mu = m < 0 ? -m : m;
    if (mu == 0) return l1 * C;
    int off = (L + 1) * C;
    for (int k = 1; k < mu; ++k) off += 2 * (L + 1 - k) * C;
    const int nm = (L + 1 - mu) * C;
    return off + (m > 0 ? 0 : nm) + (l1 - mu) * C;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_16x256(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Epilogue of one accumulator pair (o+ at tacc, o- at tacc + 128) or one
// accumulator (SIGNS = 1) holding output rows (l3, channel) for the tile's
// 128 edges, on mma.sync: per 16-edge chunk and 8 channels,
//     acc[m'][c] += sum_e D_e[+mu][m'] y+[e][c] + D_e[-mu][m'] y-[e][c],
//     y[e][c] = p_e^{head(c)} o[c][e],
// i.e. the rotate-back D^T of the |m| = mu rows weighted by the softmax and
// summed over the node's edges. A = Wigner rows (m' padded to 16, built from
// the staged fp16 pairs), B = p * o straight from tcgen05.ld.16x256b (whose
// thread layout is the mma B/D fragment layout), D = fp32 accumulators.
// Node sums go to out with fire-and-forget reductions at segment ends: one
// thread owns each (node, l3, m', c) element, so the additions happen in
// program order. The warp covers 16 TMEM lanes (channels cbase..cbase+15);
// the two warps of a lane quadrant take one half each.
template <int SIGNS>
__device__ __noinline__ void epi_mma(uint32_t tacc, int l3, int cbase, int K, int C,
                                     const __half2* __restrict__ Ds, const float* __restrict__ pch,
                                     const int* __restrict__ nb, const uint32_t* __restrict__ segm,
                                     float* __restrict__ out) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int W3 = 2 * l3 + 1, NP = npair(l3), C8 = C / 8;
    float acc[2][4];  // [n-tile lo/hi][fragment]
#pragma unroll
    for (int b2 = 0; b2 < 2; ++b2)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[b2][r] = 0.f;
    int cur = -1;
    const float* pc = pch + cbase / 8;  // 8-channel groups cbase/8 (lh = 0) and +1 (lh = 1)

    auto flush = [&]() {
        if (cur < 0) return;
#pragma unroll
        for (int lh = 0; lh < 2; ++lh)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int mp = g + ((r >> 1) << 3);
                if (mp < W3) {
                    const int c = cbase + 8 * lh + 2 * q + (r & 1);
                    atomicAdd(out + ((size_t)cur * K + l3 * l3 + mp) * C + c, acc[lh][r]);
                }
                acc[lh][r] = 0.f;
            }
    };

#pragma unroll 1
    for (int ch = 0; ch < kTileE / 16; ++ch) {
        const int e0 = ch * 16;
        // o values: [sign][edge half][4]: (c_lo,e), (c_lo,e+1), (c_hi,e), (c_hi,e+1)
        uint32_t ov[SIGNS][2][4];
#pragma unroll
        for (int s2 = 0; s2 < SIGNS; ++s2)
#pragma unroll
            for (int eh = 0; eh < 2; ++eh) tmem_ld_16x256(tacc + s2 * 128 + e0 + 8 * eh, ov[s2][eh]);
        // this thread's four edges: e0 + 2q, +1, e0 + 8 + 2q, +1
        const int ea = e0 + 2 * q, eb = e0 + 8 + 2 * q;
        // Wigner A fragments per sign: rows m' = g (a0, a2) and g + 8 (a1, a3)
        uint32_t af[SIGNS][4];
        {
            const bool r0 = g < W3, r1 = g + 8 < W3;
            const __half2 z = __float2half2_rn(0.f);
            const __half2 p00 = r0 ? Ds[ea * NP + g] : z, p01 = r0 ? Ds[(ea + 1) * NP + g] : z;
            const __half2 p10 = r1 ? Ds[ea * NP + g + 8] : z, p11 = r1 ? Ds[(ea + 1) * NP + g + 8] : z;
            const __half2 p20 = r0 ? Ds[eb * NP + g] : z, p21 = r0 ? Ds[(eb + 1) * NP + g] : z;
            const __half2 p30 = r1 ? Ds[eb * NP + g + 8] : z, p31 = r1 ? Ds[(eb + 1) * NP + g + 8] : z;
            const __half2 lo[4] = {__lows2half2(p00, p01), __lows2half2(p10, p11), __lows2half2(p20, p21),
                                   __lows2half2(p30, p31)};
#pragma unroll
            for (int k = 0; k < 4; ++k) af[0][k] = *reinterpret_cast<const uint32_t*>(&lo[k]);
            if (SIGNS == 2) {
                const __half2 hi[4] = {__highs2half2(p00, p01), __highs2half2(p10, p11), __highs2half2(p20, p21),
                                       __highs2half2(p30, p31)};
#pragma unroll
                for (int k = 0; k < 4; ++k) af[SIGNS - 1][k] = *reinterpret_cast<const uint32_t*>(&hi[k]);
            }
        }
        // softmax weights of the four edges for the two 8-channel groups
        const float2 w0 = *reinterpret_cast<const float2*>(pc + ea * C8);
        const float2 w1 = *reinterpret_cast<const float2*>(pc + (ea + 1) * C8);
        const float2 w2 = *reinterpret_cast<const float2*>(pc + eb * C8);
        const float2 w3 = *reinterpret_cast<const float2*>(pc + (eb + 1) * C8);
        const float pw[2][4] = {{w0.x, w1.x, w2.x, w3.x}, {w0.y, w1.y, w2.y, w3.y}};
        tmem_wait_ld();
        // segments of this chunk: bit k = edge e0 + k starts a node
        uint32_t bits = segm[ch];
        int lo = 0;
        if (bits & 1u) {
            flush();
            cur = nb[e0];
        }
        bits &= ~1u;
        while (true) {
            const int hi = bits ? __ffs(bits) - 1 : 16;
            // edge masks of this thread's four edges for [lo, hi)
            const float m0 = (2 * q >= lo && 2 * q < hi) ? 1.f : 0.f;
            const float m1 = (2 * q + 1 >= lo && 2 * q + 1 < hi) ? 1.f : 0.f;
            const float m2 = (8 + 2 * q >= lo && 8 + 2 * q < hi) ? 1.f : 0.f;
            const float m3 = (9 + 2 * q >= lo && 9 + 2 * q < hi) ? 1.f : 0.f;
#pragma unroll
            for (int lh = 0; lh < 2; ++lh) {
                const float* pwv = pw[lh];
#pragma unroll
                for (int s2 = 0; s2 < SIGNS; ++s2) {
                    const uint32_t* va = ov[s2][0];
                    const uint32_t* vb = ov[s2][1];
                    uint32_t bf[2];
                    bf[0] = pack_h2(pwv[0] * m0 * __uint_as_float(va[2 * lh]),
                                    pwv[1] * m1 * __uint_as_float(va[2 * lh + 1]));
                    bf[1] = pack_h2(pwv[2] * m2 * __uint_as_float(vb[2 * lh]),
                                    pwv[3] * m3 * __uint_as_float(vb[2 * lh + 1]));
                    mma_16816(acc[lh], af[s2], bf);
                }
            }
            if (hi == 16) break;
            flush();
            cur = nb[e0 + hi];
            lo = hi;
            bits &= bits - 1;
        }
    }
    flush();
}

// Wigner slice(s) a group's epilogue needs, by block (l, mu): returns bytes
// queued on `bar` into staging buffer `dst`.
// The slices (l3, |m|) of every degree of the group's rows, in increasing l3,
// one after another (the slice of degree l3 starts at pairs_in(lo, l3 - 1)).
__device__ __forceinline__ uint32_t stage_group_pairs(const TcGroup& g, int L, int C, const __half2* Dglob,
                                                      uint8_t* dst, uint64_t* bar) {
    int lo, hi;
    group_l3_range(g, L, C, lo, hi);
    const uint32_t total = (uint32_t)kTileE * 4 * pairs_in(lo, hi);
    mbar_arrive_tx(bar, total);
    for (int l3 = lo; l3 <= hi; ++l3) {
        const uint32_t bytes = (uint32_t)kTileE * npair(l3) * 4;
        bulk_load(dst, Dglob + dglob_block(l3, g.mu), bytes, bar);
        dst += bytes;
    }
    return total;
}

template <int L>
__global__ void __launch_bounds__(kThreads, 1) k_attn_tc(const __grid_constant__ TcParams P,
                                                         const __grid_constant__ TcMaps T) {
    constexpr int K = n_sh(L);
    constexpr int WS = wig_size(L);
    constexpr int DPS = dph_stride(L);
    const int C = P.C, H = P.H, dh = C / H, G = P.G, NR = P.n_rbf;
    const SmemLayout S(L, C, H, NR);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // operand tiles need 1024-byte alignment in the shared window
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* ring = smem + S.ring;
    uint8_t* dstage = smem + S.dstage;
    __half2* dph = reinterpret_cast<__half2*>(smem + S.dph);
    float* pch = reinterpret_cast<float*>(smem + S.pch);  // [2][128][C/8] softmax weight per 8 channels
    int* nid = reinterpret_cast<int*>(smem + S.nid);
    int* jn = reinterpret_cast<int*>(smem + S.jn);
    uint32_t* segm = reinterpret_cast<uint32_t*>(smem + S.segm);
    int* rpw = reinterpret_cast<int*>(smem + S.rpw);
    __half* rho = reinterpret_cast<__half*>(smem + S.rho);  // [128][16] radial basis, fp16 (gate warps)
    float* rrs = reinterpret_cast<float*>(smem + S.rrs);    // [128][16] radial basis, fp32 (logits)
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S.bars);
    uint64_t* full = bars;
    uint64_t* empty = bars + kNS;
    uint64_t* tfull = bars + 2 * kNS;
    uint64_t* tempty = tfull + 2;
    uint64_t* xready = tempty + 2;
    uint64_t* xfree = xready + 2;
    uint64_t* dbar = xfree + 2;   // epilogue Wigner staging, per buffer
    uint64_t* fin = dbar + 2;
    uint64_t* gfull = fin + 1;    // value gate of a tile buffer written (gate warps -> producer)
    uint64_t* gempty = gfull + 2; // value gate of a tile buffer consumed (producer -> gate warps)
    uint64_t* jfull = gempty + 2; // fused traversal: (i, j) of a tile buffer listed (gate warps -> producer)
    uint32_t* tmem_sm = reinterpret_cast<uint32_t*>(smem + S.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S.misc + 8);
    int* last_slot = reinterpret_cast<int*>(smem + S.misc + 16);  // producer: node slot of the last edge
    int* gij = reinterpret_cast<int*>(smem + S.misc + 64);        // gate warps: [2][128] (i, j) per edge
    long long* dsub = reinterpret_cast<long long*>(smem + S.dsub);  // sub-step cycle sums (timers on)
    float* wga = reinterpret_cast<float*>(smem + S.wga);            // [16][H] logit-gate weights
    const bool dbgon = P.dbg != nullptr;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNS; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, kEpiThreads);
            mbar_init(xready + b, 128);
            mbar_init(xfree + b, kEpiThreads);
            mbar_init(dbar + b, 1);
        }
        mbar_init(fin, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(gfull + b, 64);
            mbar_init(gempty + b, 128);
            mbar_init(jfull + b, 64);
        }
        *abort_flag = 0;
        for (int k = 0; k < 16; ++k) dsub[k] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 12) {
        tmem_alloc(tmem_sm, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_sm;


    const int n_begin = P.part[blockIdx.x], n_end = P.part[blockIdx.x + 1];
    const int e_begin = P.row_ptr[n_begin], e_end = P.row_ptr[n_end];
    const int ntiles = (e_end - e_begin + kTileE - 1) / kTileE;
    const int ng = P.n_groups;

    if (warp >= 4 && warp < 8) {
        // ---------------- producer ----------------
        const int p = threadIdx.x - 128;
        const float inv_sqrt_dh = rsqrtf((float)dh);
        const float inv_s = P.scale[1];
        const int CG = C / 8;
        const int Gv = (L + 1) * C;
        const int C8 = C / 8;
        for (int t2 = p; t2 < kTcMaxRbf * H; t2 += 128) {
            const int kb = t2 / H, h = t2 % H;
            wga[t2] = kb < NR ? P.Wrad[(size_t)kb * G + Gv + h] : 0.f;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        int nbase = n_begin;
        long long tlast = 0;
#define E2F_TICK(k)                                                   \
    do {                                                              \
        if (dbgon && p == 0) {                                        \
            const long long now_ = clock64();                         \
            dsub[k] += now_ - tlast;                                  \
            tlast = now_;                                             \
        }                                                             \
    } while (0)
        const size_t KT = (size_t)K * C;
        // L2 policies: the feature scratch is re-read by TMA (keep), neighbour rows stream (evict first)
        const uint64_t pol_last = policy_evict_last(), pol_first = policy_evict_first();
        long long w_free = 0, c_p1 = 0, c_p2 = 0;
        const long long c_start = clock64();
        for (int t = 0; t < ntiles; ++t) {
            const int b = t & 1;
            const bool okw = (t < 2) || wait_t(xfree + b, ((t - 2) >> 1) & 1, abort_flag, P.status, w_free);
            if (!bar_and(1, 128, okw)) break;
            const long long c_a = clock64();
            const int e0 = e_begin + t * kTileE;
            const int ne = min(kTileE, e_end - e0);
            // window of row_ptr after the node of the tile's first edge
            {
                int nb0;
                if (t == 0) {
                    int lo = n_begin, hi = n_end - 1;
                    while (lo < hi) {
                        int mid = (lo + hi + 1) >> 1;
                        if (P.row_ptr[mid] <= e0) lo = mid; else hi = mid - 1;
                    }
                    nb0 = lo;
                } else {
                    nb0 = *last_slot;  // node slot of edge e0 - 1
                }
                nbase = nb0;
                const int n = nbase + 1 + p;
                rpw[p] = (n <= n_end) ? P.row_ptr[n] : 0x7fffffff;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (P.cells) {
                // fused traversal: the gate warps list (atom, neighbour) of the tile's edges in
                // gij[b]; they refill it only after gempty[b], i.e. after this tile's P2
                const bool okj = wait_t(jfull + b, (t >> 1) & 1, abort_flag, P.status, w_free);
                if (!bar_and(1, 128, okj)) break;
            }
            tlast = c_a;
            E2F_TICK(0);
            __half2* Dg = P.dscr + (size_t)(blockIdx.x * 2 + b) * dglob_pairs();
            // P1: one edge per thread: frame, Wigner pairs (fp16x2; shared copy for
            // the rotation below, global copy for the epilogue), softmax weights
            {
                __half2* Dh = dph + (size_t)p * DPS;
                if (p < ne) {
                    const int e = e0 + p;
                    const int* gl = gij + b * 2 * kTileE;  // fused traversal: [i x 128][j x 128]
                    const int j = P.cells ? gl[kTileE + p] : P.col[e];
                    // node slot: last n with row_ptr[n] <= e = nbase + #{k: rpw[k] <= e}
                    int i;
                    if (e < rpw[kTileE - 1]) {
                        int lo = 0, hi = kTileE;  // first k with rpw[k] > e
                        while (lo < hi) {
                            const int mid = (lo + hi) >> 1;
                            if (rpw[mid] <= e) lo = mid + 1; else hi = mid;
                        }
                        i = nbase + lo;
                    } else {  // more than 128 nodes in reach (runs of empty rows): global search
                        int lo = nbase, hi = n_end - 1;
                        while (lo < hi) {
                            int mid = (lo + hi + 1) >> 1;
                            if (P.row_ptr[mid] <= e) lo = mid; else hi = mid - 1;
                        }
                        i = lo;
                    }
                    if (p == kTileE - 1) *last_slot = i;
                    if (P.cells) i = gl[p];  // slot -> atom
                    float3 r = edge_vec(P.pos, i, j, P.box);
                    const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
                    E2F_TICK(1);
                    float R[3][3];
                    edge_frame(r.x / d, r.y / d, r.z / d, R);
                    float D[WS];
                    wigner_blocks<L>(R, D);
                    E2F_TICK(2);
#pragma unroll
                    for (int l = 0; l <= L; ++l) {
                        const int w = 2 * l + 1;
                        const float* Dl = D + wig_off(l);
#pragma unroll
                        for (int mu = 0; mu <= l; ++mu) {
                            uint4* sq = reinterpret_cast<uint4*>(Dh + dpo(l, mu));
                            uint4* gq = reinterpret_cast<uint4*>(Dg + dglob_block(l, mu) + (size_t)p * npair(l));
#pragma unroll
                            for (int n4 = 0; n4 < npair(l); n4 += 4) {
                                uint32_t wv[4];
#pragma unroll
                                for (int t4 = 0; t4 < 4; ++t4) {
                                    const int n = n4 + t4;
                                    const float a0 = n < w ? Dl[(l + mu) * w + n] : 0.f;
                                    const float b0 = n < w ? Dl[(l - mu) * w + n] : 0.f;
                                    wv[t4] = pack_h2(a0, b0);
                                }
                                const uint4 u = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                                sq[n4 / 4] = u;
                                gq[n4 / 4] = u;
                            }
                        }
                    }
                    E2F_TICK(3);
                    float rr[kTcMaxRbf];
                    rbf_all<kTcMaxRbf>(d, P.cutoff, NR, rr);
                    {
                        float4* rq = reinterpret_cast<float4*>(rrs + p * kTcMaxRbf);
#pragma unroll
                        for (int k4 = 0; k4 < kTcMaxRbf / 4; ++k4)
                            rq[k4] = make_float4(rr[4 * k4], rr[4 * k4 + 1], rr[4 * k4 + 2], rr[4 * k4 + 3]);
                    }
                    // the neighbour's feature row is read by the rotation below: start it towards L2
                    if (p < 16)
                        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(P.x + (size_t)j * KT),
                                     "r"((uint32_t)(KT * 2))
                                     : "memory");
                    E2F_TICK(4);
                    nid[b * kTileE + p] = i;
                    jn[b * kTileE + p] = j;
                } else {
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int l = 0; l <= L; ++l)
#pragma unroll
                        for (int mu = 0; mu <= l; ++mu) {
                            uint4* gq = reinterpret_cast<uint4*>(Dg + dglob_block(l, mu) + (size_t)p * npair(l));
                            for (int n4 = 0; n4 < npair(l); n4 += 4) gq[n4 / 4] = z;
                        }
                    for (int a = 0; a < DPS; a += 4) *reinterpret_cast<uint4*>(Dh + a) = z;
                    for (int k8 = 0; k8 < C8; ++k8) pch[(b * kTileE + p) * C8 + k8] = 0.f;
                    nid[b * kTileE + p] = -1;
                    jn[b * kTileE + p] = 0;
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            E2F_TICK(6);
            // logits and softmax weights, one (edge, head) pair per thread and step: the
            // thread's head h = p % H is fixed (H divides 128), the H lanes of an edge read
            // its key row as consecutive float4
            {
                const int h = p % H, d4 = dh / 4;
                float wh[kTcMaxRbf];
#pragma unroll
                for (int kb = 0; kb < kTcMaxRbf; ++kb) wh[kb] = wga[kb * H + h];
#pragma unroll 2
                for (int e = p / H; e < ne; e += kTileE / H) {
                    const int i = nid[b * kTileE + e], j = jn[b * kTileE + e];
                    const float4* rq = reinterpret_cast<const float4*>(rrs + e * kTcMaxRbf);
                    float ga = 0.f;
#pragma unroll
                    for (int k4 = 0; k4 < kTcMaxRbf / 4; ++k4) {
                        const float4 r4 = rq[k4];
                        ga = fmaf(r4.x, wh[4 * k4], ga);
                        ga = fmaf(r4.y, wh[4 * k4 + 1], ga);
                        ga = fmaf(r4.z, wh[4 * k4 + 2], ga);
                        ga = fmaf(r4.w, wh[4 * k4 + 3], ga);
                    }
                    const float4* q4 = reinterpret_cast<const float4*>(P.q + (size_t)i * C + h * dh);
                    const float4* k4 = reinterpret_cast<const float4*>(P.k + (size_t)j * C + h * dh);
                    float dot = 0.f;
                    for (int c4 = 0; c4 < d4; ++c4) {
                        const float4 qa = __ldg(q4 + c4), kv = __ldg(k4 + c4);
                        dot = fmaf(qa.x, kv.x, dot);
                        dot = fmaf(qa.y, kv.y, dot);
                        dot = fmaf(qa.z, kv.z, dot);
                        dot = fmaf(qa.w, kv.w, dot);
                    }
                    const float a = ga * dot * inv_sqrt_dh;
                    const float pw = expf(a - P.lse[(size_t)i * H + h]) * inv_s;
                    for (int k8 = h * (dh / 8); k8 < (h + 1) * (dh / 8); ++k8) pch[(b * kTileE + e) * C8 + k8] = pw;
                }
            }
            E2F_TICK(5);
            if (p < kTileE / kChunk) {  // segment starts per 16-edge chunk
                uint32_t m = 0;
                for (int q = 0; q < kChunk; ++q) {
                    const int e = p * kChunk + q;
                    if (e == 0 || nid[b * kTileE + e] != nid[b * kTileE + e - 1]) m |= 1u << q;
                }
                segm[b * (kTileE / kChunk) + p] = m;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            E2F_TICK(7);
            const long long c_b = clock64();
            c_p1 += c_b - c_a;
            // P2: rotated, gated features -> scratch row (e), all |m| blocks (fp16, packed math)
            {
                const bool okg = wait_t(gfull + b, (t >> 1) & 1, abort_flag, P.status, w_free);
                if (!bar_and(1, 128, okg)) break;
            }
            const __half* gs = P.gscr + ((size_t)blockIdx.x * 2 + b) * kTileE * Gv;
            __half* xrow0 = P.xs + ((size_t)(blockIdx.x * 2 + b) * kTileE) * KT;
            for (int it = p; it < kTileE * CG; it += 128) {
                const int e = it / CG, c0 = (it % CG) * 8;
                __half* xrow = xrow0 + (size_t)e * KT;
                if (e >= ne) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int l1 = 0; l1 <= L; ++l1)
#pragma unroll
                        for (int m = -l1; m <= l1; ++m)
                            *reinterpret_cast<uint4*>(xrow + kpos(l1, m, L, C) + c0) = z;
                    continue;
                }
                const int j = jn[b * kTileE + e];
                if (c0 == 0 && e + 16 < ne)  // neighbour row of the edge two rounds ahead
                    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                                     P.x + (size_t)jn[b * kTileE + e + 16] * KT),
                                 "r"((uint32_t)(KT * 2))
                                 : "memory");
                const __half2* De = dph + (size_t)e * DPS;
                // all (L+1)^2 rows of x_j for these 8 channels in flight at once
                uint4 raw[K];
                const __half* xj = P.x + (size_t)j * K * C + c0;
#pragma unroll
                for (int n = 0; n < K; ++n) raw[n] = ld_hint(xj + (size_t)n * C, pol_first);
                uint4 gr[L + 1];
#pragma unroll
                for (int l1 = 0; l1 <= L; ++l1) gr[l1] = *reinterpret_cast<const uint4*>(gs + (size_t)e * Gv + l1 * C + c0);
#pragma unroll
                for (int l1 = 0; l1 <= L; ++l1) {
                    constexpr int kMaxW = 2 * kMaxL + 1;
                    const int w = 2 * l1 + 1;
                    const __half2* g2 = reinterpret_cast<const __half2*>(&gr[l1]);
                    __half2 xs2[kMaxW][4];
#pragma unroll
                    for (int n = 0; n < kMaxW; ++n) {
                        if (n < w) {
                            const __half2* h2 = reinterpret_cast<const __half2*>(&raw[l1 * l1 + n]);
#pragma unroll
                            for (int q = 0; q < 4; ++q) xs2[n][q] = __hmul2(h2[q], g2[q]);
                        }
                    }
#pragma unroll
                    for (int mu = 0; mu <= kMaxL; ++mu) {
                        if (mu <= l1) {
                            const __half2* Dq = De + dpo(l1, mu);
                            __half2 op[4], om[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) { op[q] = __float2half2_rn(0.f); om[q] = op[q]; }
#pragma unroll
                            for (int n = 0; n < kMaxW; ++n) {
                                if (n < w) {
                                    const __half2 pr = Dq[n];
                                    const __half2 dp = __low2half2(pr), dm = __high2half2(pr);
#pragma unroll
                                    for (int q = 0; q < 4; ++q) {
                                        op[q] = __hfma2(dp, xs2[n][q], op[q]);
                                        om[q] = __hfma2(dm, xs2[n][q], om[q]);
                                    }
                                }
                            }
                            st_hint(xrow + kpos(l1, mu, L, C) + c0, *reinterpret_cast<uint4*>(op), pol_last);
                            if (mu > 0)
                                st_hint(xrow + kpos(l1, -mu, L, C) + c0, *reinterpret_cast<uint4*>(om), pol_last);
                        }
                    }
                }
            }
            mbar_arrive(gempty + b);  // this tile's value gates have been read
            // generic-proxy stores (features, Wigner pairs) -> visible to TMA / bulk copies
            asm volatile("fence.proxy.async.global;" ::: "memory");
            // (test hook: CTA 0 withholds one arrival on its first tile, so that the
            // bounded waits on xready run out and the CTA takes its abort path)
            if (!(P.drop_arrive && blockIdx.x == 0 && t == 0 && p == 0)) mbar_arrive(xready + b);
            c_p2 += clock64() - c_b;
        }
        if (P.dbg && p == 0) {
            long long* d = P.dbg + blockIdx.x * kDbgSlots;
            d[0] = w_free; d[1] = clock64() - c_start; d[11] = c_p1; d[12] = c_p2;
            for (int k = 0; k < 8; ++k) d[14 + k] = dsub[k];
        }
#undef E2F_TICK
    } else if (warp == 12) {
        // ---------------- TMA ----------------
        if (lane == 0) {
            const uint64_t pol_xs = policy_evict_last();
            int stage = 0;
            uint32_t ph = 0;
            bool ok = true;
            int pending[kNS];
            for (int s2 = 0; s2 < kNS; ++s2) pending[s2] = -1;
            long long w_x = 0, w_e = 0;
            const long long c_start = clock64();
            for (int t = 0; t < ntiles && ok; ++t) {
                const int b = t & 1;
                if (!wait_t(xready + b, (t >> 1) & 1, abort_flag, P.status, w_x)) { ok = false; break; }
                const int rowT = (blockIdx.x * 2 + b) * kTileE;
                for (int gi = 0; gi < ng && ok; ++gi) {
                    const TcGroup g = P.groups[gi];
                    for (int kk = 0; kk < g.klen; kk += kKS) {
                        if (!wait_t(empty + stage, ph ^ 1, abort_flag, P.status, w_e)) { ok = false; break; }
                        uint8_t* st = ring + (size_t)stage * kStage;
                        const int ntile = g.mu > 0 ? 4 : (g.row0b >= 0 ? 3 : 2);
                        mbar_arrive_tx(full + stage, ntile * kSlot);
                        if (g.mu > 0) {
                            tma_load_2d(st, &T.w[g.wa], kk, g.row0, full + stage);
                            tma_load_2d(st + kSlot, &T.w[g.wb], kk, g.row0, full + stage);
                            tma_load_2d_hint(st + 2 * kSlot, &T.xs, g.xoff0 + kk, rowT, full + stage, pol_xs);
                            tma_load_2d_hint(st + 3 * kSlot, &T.xs, g.xoff1 + kk, rowT, full + stage, pol_xs);
                        } else {
                            tma_load_2d(st, &T.w[g.wa], kk, g.row0, full + stage);
                            if (g.row0b >= 0) tma_load_2d(st + kSlot, &T.w[g.wa], kk, g.row0b, full + stage);
                            tma_load_2d_hint(st + 2 * kSlot, &T.xs, g.xoff0 + kk, rowT, full + stage, pol_xs);
                        }
                        pending[stage] = (int)ph;
                        if (++stage == kNS) { stage = 0; ph ^= 1; }
                    }
                }
            }
            if (P.dbg) {
                long long* d = P.dbg + blockIdx.x * kDbgSlots;
                d[2] = w_x; d[3] = w_e; d[4] = clock64() - c_start;
            }
            // every issued load lands (bounded wait) before the CTA can leave
            for (int s2 = 0; s2 < kNS; ++s2) {
                if (pending[s2] < 0) continue;
                const uint64_t t0 = gtimer();
                while (!mbar_try(full + s2, (uint32_t)pending[s2]) && gtimer() - t0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 13) {
        // ---------------- MMA ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t ph = 0;
            long long gcount = 0;
            bool ok = true;
            long long w_t = 0, w_f = 0;
            const long long c_start = clock64();
            constexpr uint32_t ID = idesc_f16(false), IDN = idesc_f16(true);
            for (int t = 0; t < ntiles && ok; ++t) {
                for (int gi = 0; gi < ng && ok; ++gi, ++gcount) {
                    const TcGroup g = P.groups[gi];
                    const int slot = (int)(gcount & 1);
                    const uint32_t use = (uint32_t)(gcount >> 1);
                    if (!wait_t(tempty + slot, (use & 1) ^ 1, abort_flag, P.status, w_t)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d0 = tmem + slot * 256, d1 = d0 + 128;
                    for (int kk = 0; kk < g.klen; kk += kKS) {
                        if (!wait_t(full + stage, ph, abort_flag, P.status, w_f)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(ring + (size_t)stage * kStage);
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {
                            const uint64_t a0 = sdesc_sw64(sa + ks * 32);
                            const uint64_t a1 = sdesc_sw64(sa + kSlot + ks * 32);
                            const uint64_t x0 = sdesc_sw64(sa + 2 * kSlot + ks * 32);
                            const uint64_t x1 = sdesc_sw64(sa + 3 * kSlot + ks * 32);
                            const uint32_t acc = (kk > 0 || ks > 0) ? 1u : 0u;
                            if (g.mu > 0) {
                                umma(d0, a0, x0, ID, acc);    // o+ += A h+
                                umma(d1, a1, x0, ID, acc);    // o- += B h+
                                umma(d0, a1, x1, IDN, 1u);    // o+ -= B h-
                                umma(d1, a0, x1, ID, 1u);     // o- += A h-
                            } else {
                                umma(d0, a0, x0, ID, acc);
                                if (g.row0b >= 0) umma(d1, a1, x0, ID, acc);
                            }
                        }
                        umma_commit(empty + stage);
                        if (++stage == kNS) { stage = 0; ph ^= 1; }
                    }
                    if (ok) umma_commit(tfull + slot);
                }
            }
            if (P.dbg) {
                long long* d = P.dbg + blockIdx.x * kDbgSlots;
                d[5] = w_t; d[6] = w_f; d[7] = clock64() - c_start;
            }
            // every issued MMA completes (bounded wait) before TMEM is released
            umma_commit(fin);
            const uint64_t t0 = gtimer();
            while (!mbar_try(fin, 0) && gtimer() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else if (warp >= 14) {
        // ---------------- value gate (warps 14-15), up to two tiles ahead ----------------
        // g[e][n] = rho(d_e) . W_rad[:, n] for the tile's 128 edges and n < (L+1)C, into a
        // per-CTA global buffer per tile parity that the producer's rotation reads.
        const int gp = threadIdx.x - 448, gw = warp - 14, g8 = lane >> 2, t4 = lane & 3;
        const int Gv = (L + 1) * C;
        long long w_g = 0;
        const long long c_start = clock64();
        for (int t = 0; t < ntiles; ++t) {
            const int b = t & 1;
            const bool okw = (t < 2) || wait_t(gempty + b, ((t - 2) >> 1) & 1, abort_flag, P.status, w_g);
            if (!bar_and(3, 64, okw)) break;
            const int e0 = e_begin + t * kTileE;
            const int ne = min(kTileE, e_end - e0);
            int* gi = gij + b * 2 * kTileE;
            if (P.cells) {  // fused traversal: (atom, neighbour) of each edge from the cell lists
                auto slot_of = [&](int e) {
                    int lo = n_begin, hi = n_end - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (P.row_ptr[mid] <= e) lo = mid; else hi = mid - 1;
                    }
                    return lo;
                };
                const int s_first = slot_of(e0), s_last = slot_of(e0 + ne - 1);
                for (int sl = s_first + (warp - 14); sl <= s_last; sl += 2) {
                    const int base = P.row_ptr[sl], ia = P.cv.sidx[sl];
                    warp_neighbors(
                        P.cv, P.cv.spos[sl], ia,
                        [&](int k, int j) {
                            const int e = base + k;
                            if (e >= e0 && e < e0 + ne) {
                                gi[e - e0] = ia;
                                gi[kTileE + e - e0] = j;
                            }
                        },
                        0, sl);
                }
                asm volatile("bar.sync 3, 64;" ::: "memory");
                mbar_arrive(jfull + b);  // releases the lists to the producer (CTA scope)
            }
            for (int k = gp; k < kTileE; k += 64) {  // radial basis of the tile's edges
                float rr[kTcMaxRbf];
                if (k < ne) {
                    const int e = e0 + k;
                    int lo, j;
                    if (P.cells) {
                        lo = gi[k];
                        j = gi[kTileE + k];
                    } else {
                        j = P.col[e];
                        lo = n_begin;
                        int hi = n_end - 1;  // node i: last n with row_ptr[n] <= e
                        while (lo < hi) {
                            const int mid = (lo + hi + 1) >> 1;
                            if (P.row_ptr[mid] <= e) lo = mid; else hi = mid - 1;
                        }
                    }
                    const float3 r = edge_vec(P.pos, lo, j, P.box);
                    const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
                    rbf_all<kTcMaxRbf>(d, P.cutoff, NR, rr);
                } else {
#pragma unroll
                    for (int kb = 0; kb < kTcMaxRbf; ++kb) rr[kb] = 0.f;
                }
                uint32_t hw[kTcMaxRbf / 2];
#pragma unroll
                for (int kb = 0; kb < kTcMaxRbf / 2; ++kb) hw[kb] = pack_h2(rr[2 * kb], rr[2 * kb + 1]);
                uint4* rq = reinterpret_cast<uint4*>(rho + k * kTcMaxRbf);
                rq[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                rq[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
            }
            asm volatile("bar.sync 3, 64;" ::: "memory");
            // one k = 16 mma.sync per 16 edges x 8 columns; warp gw takes edge blocks 4 gw .. 4 gw + 3
            __half* gs = P.gscr + ((size_t)blockIdx.x * 2 + b) * kTileE * Gv;
            uint32_t af[4][4];
#pragma unroll
            for (int mb = 0; mb < 4; ++mb) {
                const __half* rr0 = rho + ((4 * gw + mb) * 16 + g8) * kTcMaxRbf + 2 * t4;
                af[mb][0] = *reinterpret_cast<const uint32_t*>(rr0);
                af[mb][1] = *reinterpret_cast<const uint32_t*>(rr0 + 8 * kTcMaxRbf);
                af[mb][2] = *reinterpret_cast<const uint32_t*>(rr0 + 8);
                af[mb][3] = *reinterpret_cast<const uint32_t*>(rr0 + 8 * kTcMaxRbf + 8);
            }
#pragma unroll 2
            for (int n0 = 0; n0 < Gv; n0 += 8) {
                const __half* wb = P.whT + (size_t)(n0 + g8) * kTcMaxRbf + 2 * t4;
                uint32_t bf[2];
                bf[0] = __ldg(reinterpret_cast<const unsigned int*>(wb));
                bf[1] = __ldg(reinterpret_cast<const unsigned int*>(wb + 8));
#pragma unroll
                for (int mb = 0; mb < 4; ++mb) {
                    float acc4[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_16816(acc4, af[mb], bf);
                    const int e = (4 * gw + mb) * 16 + g8;
                    *reinterpret_cast<__half2*>(gs + (size_t)e * Gv + n0 + 2 * t4) = __floats2half2_rn(acc4[0], acc4[1]);
                    *reinterpret_cast<__half2*>(gs + (size_t)(e + 8) * Gv + n0 + 2 * t4) =
                        __floats2half2_rn(acc4[2], acc4[3]);
                }
            }
            mbar_arrive(gfull + b);  // releases the stores above to the producer (CTA scope)
        }
        if (P.dbg && gp == 0) {
            long long* d = P.dbg + blockIdx.x * kDbgSlots;
            d[23] = w_g; d[24] = clock64() - c_start;
        }
    } else if (warp < 12) {
        // ---------------- epilogue (warps 0-3 and 8-11) ----------------
        // Every decision to stop goes through bar_and, so the 128 threads leave
        // together and no thread is left at a named barrier.
        const int r = threadIdx.x;
        long long gcount = 0;
        bool ok = true;
        long long w_x = 0, w_t = 0;
        long long staged[2] = {-1, -1};  // last group index staged into each buffer (thread 0)
        const long long c_start = clock64();
        for (int t = 0; t < ntiles; ++t) {
            const int b = t & 1;
            const bool okx = wait_t(xready + b, (t >> 1) & 1, abort_flag, P.status, w_x);
            if (!bar_and(2, kEpiThreads, ok && okx)) { ok = false; break; }
            const __half2* Dg = P.dscr + (size_t)(blockIdx.x * 2 + b) * dglob_pairs();
            const float* pb = pch + (size_t)b * kTileE * (C / 8);
            const int* nb = nid + b * kTileE;
            const uint32_t* sg = segm + b * (kTileE / kChunk);
            if (r == 0) {
                stage_group_pairs(P.groups[0], L, C, Dg, dstage + (gcount & 1) * S.dstride, dbar + (gcount & 1));
                staged[gcount & 1] = gcount;
            }
            for (int gi = 0; gi < ng; ++gi, ++gcount) {
                // all threads are done with group gcount-1, so its staging buffer can be refilled
                if (!bar_and(2, kEpiThreads, ok)) { ok = false; break; }
                if (r == 0 && gi + 1 < ng) {
                    stage_group_pairs(P.groups[gi + 1], L, C, Dg, dstage + ((gcount + 1) & 1) * S.dstride,
                                      dbar + ((gcount + 1) & 1));
                    staged[(gcount + 1) & 1] = gcount + 1;
                }
                const TcGroup g = P.groups[gi];
                const int slot = (int)(gcount & 1);
                const uint32_t use = (uint32_t)(gcount >> 1);
                const bool okd = wait_t(dbar + slot, use & 1, abort_flag, P.status, w_t);
                const bool okt = okd && wait_t(tfull + slot, use & 1, abort_flag, P.status, w_t);
                if (okt) {
                    const long long c_e0 = clock64();
                    tc_fence_after();
                    const __half2* Ds = reinterpret_cast<const __half2*>(dstage + slot * S.dstride);
                    const int lrow = (warp & 3) * 32 + (warp >> 3) * 16;  // this warp's 16 TMEM lanes
                    const uint32_t twarp = tmem + ((uint32_t)lrow << 16) + slot * 256;
                    int lo, hi;
                    group_l3_range(g, L, C, lo, hi);
                    // rows of this warp: one l3, 16 channels; rows past degree L are padding
                    if (g.mu > 0) {
                        const int row = g.row0 + lrow, l3 = g.mu + row / C;
                        if (l3 <= L)
                            epi_mma<2>(twarp, l3, row % C, K, C, Ds + kTileE * pairs_in(lo, l3 - 1), pb, nb, sg, P.out);
                    } else {
                        const int ra = g.row0 + lrow, la = ra / C;
                        if (la <= L)
                            epi_mma<1>(twarp, la, ra % C, K, C, Ds + kTileE * pairs_in(lo, la - 1), pb, nb, sg, P.out);
                        if (g.row0b >= 0) {
                            const int rb = g.row0b + lrow, lb = rb / C;
                            if (lb <= L)
                                epi_mma<1>(twarp + 128, lb, rb % C, K, C, Ds + kTileE * pairs_in(lo, lb - 1), pb, nb, sg,
                                           P.out);
                        }
                    }
                    tc_fence_before();
                    if (dbgon && r == 0) dsub[8] += clock64() - c_e0;
                } else {
                    ok = false;
                }
                mbar_arrive(tempty + slot);
            }
            if (!bar_and(2, kEpiThreads, ok)) { ok = false; break; }
            mbar_arrive(xfree + b);
        }
        if (P.dbg && r == 0) {
            long long* d = P.dbg + blockIdx.x * kDbgSlots;
            d[8] = w_x; d[9] = w_t; d[10] = clock64() - c_start; d[13] = ntiles; d[22] = dsub[8];
        }
        // a staging copy that was issued but never waited for lands before exit
        if (r == 0) {
            for (int s2 = 0; s2 < 2; ++s2) {
                if (staged[s2] < 0) continue;
                const uint64_t t0 = gtimer();
                while (!mbar_try(dbar + s2, (uint32_t)((staged[s2] >> 1) & 1)) && gtimer() - t0 < kWaitNs) {
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 12) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tc

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)tc::kKS, 128};
    cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(int L, int C, int H, int n_rbf, bool bf16) {
    return bf16 && L >= 1 && L <= kMaxL && (C % 128 == 0 || C == 64) && C <= 256 && H <= kMaxHeads && H % 4 == 0 &&
           C % H == 0 && (C / H) % 8 == 0 &&
           n_rbf <= kTcMaxRbf && tc::SmemLayout(L, C, H, n_rbf).total + 1024 <= 232448;
}

namespace {
struct TcWs {
    size_t dbg, lse, part, xs, dscr, x16, w16, whT, gscr, words, total;
    TcWs(int64_t n_atoms, int L, int C, int H) {
        const int K = n_sh(L), Gv = (L + 1) * C;
        size_t o = 0;
        auto take = [&](size_t b) { size_t r = o; o = align_up(o + b, 256); return r; };
        dbg = take(kTcDebugBytes);
        lse = take(4 * (size_t)n_atoms * H);
        part = take(4 * (size_t)(kMaxCtas + 1));
        xs = take((size_t)kMaxCtas * 2 * tc::kTileE * K * C * 2);
        dscr = take((size_t)kMaxCtas * 2 * tc::dglob_pairs() * 4);
        x16 = take((size_t)n_atoms * K * C * 2);
        w16 = take(so2_total(L, C) * 2);
        whT = take((size_t)Gv * kTcMaxRbf * 2);
        gscr = take((size_t)kMaxCtas * 2 * tc::kTileE * Gv * 2);  // two tile buffers per CTA
        words = take(256);
        total = o;
    }
};
}  // namespace

size_t tc_workspace_bytes(int64_t n_atoms, int L, int C, int H) { return TcWs(n_atoms, L, C, H).total; }

namespace {
// caller events recorded around the main kernel (profiling aid; see
// e2f_attention_set_kernel_events)
cudaEvent_t g_kernel_ev[2] = {nullptr, nullptr};
// debug and test controls (set_tc_debug)
int g_dbg_max_ctas = 0, g_dbg_timers = 0, g_dbg_drop = 0;
}  // namespace

void set_tc_kernel_events(void* start, void* stop) {
    g_kernel_ev[0] = static_cast<cudaEvent_t>(start);
    g_kernel_ev[1] = static_cast<cudaEvent_t>(stop);
}

void set_tc_debug(int max_ctas, int timers, int drop_arrive) {
    g_dbg_max_ctas = max_ctas;
    g_dbg_timers = timers;
    g_dbg_drop = drop_arrive;
}

template <int L>
static cudaError_t launch_tc(const tc::TcParams& P, const tc::TcMaps& T, int grid, cudaStream_t s) {
    const size_t smem = tc::SmemLayout(L, P.C, P.H, P.n_rbf).total + 1024;
    cudaError_t e = cudaFuncSetAttribute(tc::k_attn_tc<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    tc::k_attn_tc<L><<<grid, tc::kThreads, smem, s>>>(P, T);
    return cudaGetLastError();
}

cudaError_t run_attention_tc(const AttnArgs& a, void* tc_ws, cudaStream_t s, const CellLists* cl) {
    const int L = a.L, C = a.C, H = a.H, K = n_sh(L), N = a.n_atoms;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    int cap = kMaxCtas;
    if (g_dbg_max_ctas > 0 && g_dbg_max_ctas < cap) cap = g_dbg_max_ctas;  // fewer, longer CTAs (tests)
    const int grid = std::max(1, std::min(sms, cap));
    const TcWs Wl(N, L, C, H);
    char* w = static_cast<char*>(tc_ws);
    long long* dbg = reinterpret_cast<long long*>(w + Wl.dbg);
    float* lse = reinterpret_cast<float*>(w + Wl.lse);
    int32_t* part = reinterpret_cast<int32_t*>(w + Wl.part);
    __half* xs = reinterpret_cast<__half*>(w + Wl.xs);
    __half2* dscr = reinterpret_cast<__half2*>(w + Wl.dscr);
    __half* x16 = reinterpret_cast<__half*>(w + Wl.x16);
    __half* w16 = reinterpret_cast<__half*>(w + Wl.w16);
    __half* whT = reinterpret_cast<__half*>(w + Wl.whT);
    __half* gscr = reinterpret_cast<__half*>(w + Wl.gscr);
    unsigned* amax = reinterpret_cast<unsigned*>(w + Wl.words);
    float* scale = reinterpret_cast<float*>(w + Wl.words + 16);
    const int G = (L + 1) * C + H, Gv = (L + 1) * C;

    // fp16 operands: feature scale, scaled features, weights
    e = cudaMemsetAsync(amax, 0, 16, s);
    if (e != cudaSuccess) return e;
    const size_t nx = (size_t)N * K * C;
    count_launch();
    tc::k_amax<<<592, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.x), nx, a.Wrad, (size_t)a.n_rbf * G, amax);
    count_launch();
    tc::k_make_scale<<<1, 1, 0, s>>>(amax, a.n_rbf, scale, a.status);
    count_launch();
    tc::k_x_to_f16<<<1184, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.x), nx, scale, x16);
    count_launch();
    tc::k_w_to_f16<<<592, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.Wso2), so2_total(L, C, a.M), w16);
    count_launch();
    tc::k_wrad_t<<<(Gv * kTcMaxRbf + 255) / 256, 256, 0, s>>>(a.Wrad, a.n_rbf, G, Gv, whT);

    // pre-passes: Q/K, softmax statistics, partition, zeroed output
    count_launch();
    tc::k_qk_tiled<<<dim3((N + tc::kQkM - 1) / tc::kQkM, (2 * C + tc::kQkN - 1) / tc::kQkN), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(a.x), N, K, C, a.Wq, a.Wk, a.q, a.k);
    StatsParams sp{};
    sp.n_atoms = N; sp.C = C; sp.H = H; sp.n_rbf = a.n_rbf; sp.G = (L + 1) * C + H; sp.cutoff = a.cutoff;
    sp.box = a.box; sp.pos = a.pos; sp.row_ptr = a.row_ptr; sp.col = a.col; sp.q = a.q; sp.k = a.k;
    sp.Wrad = a.Wrad; sp.lse = lse;
    count_launch();
    if (cl) {
        tc::k_softmax_stats_cells<<<(N + 7) / 8, 256, 0, s>>>(sp, cl->view);
        count_launch();
        tc::k_flags_to_status<<<1, 1, 0, s>>>(cl->flags, a.status);
    } else {
        tc::k_softmax_stats<<<(N + 7) / 8, 256, 0, s>>>(sp);
    }
    count_launch();
    tc::k_partition<<<(grid + 1 + 127) / 128, 128, 0, s>>>(a.row_ptr, N, grid, part);
    e = cudaMemsetAsync(a.out, 0, (size_t)N * K * C * 4, s);
    if (e != cudaSuccess) return e;

    tc::TcParams P{};
    P.C = C; P.H = H; P.n_rbf = a.n_rbf; P.G = (L + 1) * C + H; P.M = a.M; P.cutoff = a.cutoff; P.box = a.box;
    P.pos = a.pos; P.row_ptr = a.row_ptr; P.col = a.col; P.x = x16; P.whT = whT; P.gscr = gscr; P.scale = scale;
    P.q = a.q; P.k = a.k; P.lse = lse; P.Wrad = a.Wrad; P.part = part; P.xs = xs; P.dscr = dscr; P.out = a.out;
    P.status = a.status;
    P.cells = cl ? 1 : 0;
    if (cl) P.cv = cl->view;
    P.dbg = nullptr;
    if (g_dbg_timers) {
        P.dbg = dbg;
        e = cudaMemsetAsync(dbg, 0, kTcDebugBytes, s);
        if (e != cudaSuccess) return e;
    }
    P.drop_arrive = g_dbg_drop ? 1 : 0;
    // groups: m = 0 feature blocks in pairs; then (o+, o-) pairs per block for m >= 1
    int ng = 0;
    const int n0 = (L + 1) * C;
    for (int r0 = 0; r0 < n0; r0 += 256) {
        tc::TcGroup g{};
        g.mu = 0; g.row0 = r0; g.row0b = (r0 + 128 < n0) ? r0 + 128 : -1; g.klen = n0; g.xoff0 = 0; g.xoff1 = 0;
        g.wa = 0; g.wb = 0;
        P.groups[ng++] = g;
    }
    int koff = n0;
    for (int mu = 1; mu <= a.M; ++mu) {  // |m| > M: no message (truncated layer)
        const int nm = (L + 1 - mu) * C;
        for (int r0 = 0; r0 < nm; r0 += 128) {
            tc::TcGroup g{};
            g.mu = mu; g.row0 = r0; g.row0b = -1; g.klen = nm; g.xoff0 = koff; g.xoff1 = koff + nm;
            g.wa = 2 * mu - 1; g.wb = 2 * mu;
            P.groups[ng++] = g;
        }
        koff += 2 * nm;
    }
    P.n_groups = ng;

    tc::TcMaps T;
    const __half* W = w16;
    if (!make_map(&T.w[0], W + so2_offset(L, C, 0, 0), n0, n0)) return cudaErrorInvalidValue;
    for (int mu = 1; mu <= a.M; ++mu) {
        const int nm = (L + 1 - mu) * C;
        if (!make_map(&T.w[2 * mu - 1], W + so2_offset(L, C, mu, 0), nm, nm)) return cudaErrorInvalidValue;
        if (!make_map(&T.w[2 * mu], W + so2_offset(L, C, mu, 1), nm, nm)) return cudaErrorInvalidValue;
    }
    if (!make_map(&T.xs, xs, (uint64_t)K * C, (uint64_t)grid * 2 * tc::kTileE)) return cudaErrorInvalidValue;

    if (g_kernel_ev[0] && g_kernel_ev[1]) {
        e = cudaEventRecord(g_kernel_ev[0], s);
        if (e != cudaSuccess) return e;
        switch (L) {
            case 1: e = launch_tc<1>(P, T, grid, s); break;
            case 2: e = launch_tc<2>(P, T, grid, s); break;
            case 3: e = launch_tc<3>(P, T, grid, s); break;
            case 4: e = launch_tc<4>(P, T, grid, s); break;
            default: return cudaErrorInvalidValue;
        }
        if (e != cudaSuccess) return e;
        return cudaEventRecord(g_kernel_ev[1], s);
    }
    switch (L) {
        case 1: return launch_tc<1>(P, T, grid, s);
        case 2: return launch_tc<2>(P, T, grid, s);
        case 3: return launch_tc<3>(P, T, grid, s);
        case 4: return launch_tc<4>(P, T, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace e2f
