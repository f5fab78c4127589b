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
//   0-3        epilogue (warp w: TMEM lanes 32w..32w+31): converts a group's
//              accumulators in place to fp16 p * o (p = softmax weight of the
//              edge and the row's head), builds per-node Wigner operand blocks
//              and drains the rotate-back results D2 = (p o) D into out[node]
//              (one owner thread per element: fixed order)
//   4-7        producer: per edge the node, frame, Wigner blocks (fp16 pairs,
//              shared and global copies); per (edge, head) the softmax weight
//              p = exp(a - lse) (statistics from an O(N) pre-pass); per
//              (edge, 8 channels) the gathered, gated, rotated features,
//              written once per tile to a per-CTA global scratch row for TMA
//   8, 13      tcgen05.mma issue (one thread each): warp 13 the first
//              accumulator of a group and the rotate-back MMAs (A operand in
//              TMEM) of the previous group, warp 8 the second accumulator
//   12         TMA loads of weight and feature tiles into a 3-stage ring
//   14-15      value gates rho(d) W_rad of a tile (mma.sync), up to two tiles
//              ahead of the producer, into a double-buffered global scratch
//   9-11       idle
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

// Q/K projection, 32 nodes per CTA, weights staged in shared memory in blocks
// of 64 output channels.
constexpr int kQkRows = 64;
__global__ void __launch_bounds__(256) k_qk_tiled(const __nv_bfloat16* __restrict__ x, int n_atoms, int K, int C,
                                                   const float* __restrict__ Wq, const float* __restrict__ Wk,
                                                   float* q, float* k) {
    extern __shared__ float sm[];
    float* xs = sm;                // [32][C]
    float* ws = xs + 32 * C;       // [kQkRows][C+1]
    const int n0 = blockIdx.x * 32;
    for (int t = threadIdx.x; t < 32 * C; t += blockDim.x) {
        const int a = t / C, c = t % C;
        xs[t] = (n0 + a < n_atoms) ? __bfloat162float(x[(size_t)(n0 + a) * K * C + c]) : 0.f;
    }
    for (int which = 0; which < 2; ++which) {
        const float* W = which ? Wk : Wq;
        float* dst = which ? k : q;
        for (int r0 = 0; r0 < C; r0 += kQkRows) {
            const int nr = min(kQkRows, C - r0);
            __syncthreads();
            for (int t = threadIdx.x; t < nr * C; t += blockDim.x)
                ws[(t / C) * (C + 1) + t % C] = W[(size_t)(r0 + t / C) * C + t % C];
            __syncthreads();
            for (int t = threadIdx.x; t < 32 * nr; t += blockDim.x) {
                const int a = t / nr, c = t % nr;
                float s = 0.f;
                for (int c2 = 0; c2 < C; ++c2) s = fmaf(ws[c * (C + 1) + c2], xs[a * C + c2], s);
                if (n0 + a < n_atoms) dst[(size_t)(n0 + a) * C + r0 + c] = s;
            }
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
constexpr int kTileE = 128;                   // edges of a pair tile (MMA N)
constexpr int kHalfE = 64;                    // edges of a pair tile held by each CTA
constexpr int kKS = 32;                       // K per ring stage
constexpr int kNS = 5;                        // ring stages
constexpr int kWSlot = 128 * kKS * 2;         // 8 KB weight tile (128 rows of this CTA)
constexpr int kXSlot = kHalfE * kKS * 2;      // 4 KB feature tile (this CTA's 64 edges)
constexpr int kStage = 2 * kWSlot + 2 * kXSlot;
constexpr int kThreads = 512;
constexpr int kEpiThreads = 128;

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
// global copy (epilogue), per CTA and tile buffer, block-major: block (l, mu)
// holds npair(l) x the CTA's 64 edges (pair index outer, edge inner), so each
// CTA's part of a group's slice is one bulk copy and the epilogue reads a
// pair for 8 consecutive edges with two 16-byte loads
__host__ __device__ constexpr size_t dglob_pairs() { return (size_t)kHalfE * dptotal(kMaxL); }
__host__ __device__ constexpr size_t dglob_block(int l, int mu) { return (size_t)kHalfE * dpo(l, mu); }
static_assert(npair(0) == 4 && npair(1) == 4 && npair(2) == 8 && npair(3) == 8 && npair(4) == 12, "pairs");
static_assert(dptotal(4) == 128, "pair layout");

// Bytes of Wigner pairs one group's epilogue stages in a CTA: npair(l)
// pairs of 4 bytes per edge of the pair tile for each of the CTA's one or two
// accumulators (their degrees may differ).
__host__ __device__ inline size_t stage_bytes(int L, int C) {
    (void)C;
    return (size_t)kTileE * 4 * 2 * npair(L);
}

// Rotate-back contraction on the tensor cores (see the epilogue): per pass at
// most kB2Blocks operand blocks of 16 rows (m') x 16 edges, fp16.
constexpr int kB2Blocks = 24;  // per buffer; two buffers
constexpr int kB2Bytes = 512;  // this CTA's 16 rows (m') x 16 edges of a 32-row pair operand

// Shared memory layout (bytes), shared by host (size) and device (offsets).
struct SmemLayout {
    size_t ring, dstage, dstride, dph, php, nid, jn, rpw, rho, rrs, wga, b2, slots, req, bars, misc, dsub, total;
    __host__ __device__ SmemLayout(int L, int C, int H, int n_rbf) {
        size_t o = 0;
        ring = o;   o += (size_t)kNS * kStage;
        dstride = (stage_bytes(L, C) + 127) & ~size_t(127);
        dstage = o; o += 2 * dstride;
        dph = o;    o += (size_t)kHalfE * dph_stride(L) * 4;
        php = o;    o += 2ull * H * kTileE * 4;          // [2][H][128] softmax weight per head and pair-tile edge
        nid = o;    o += 2ull * kTileE * 4;              // [2][128] node of each pair-tile edge
        jn = o;     o += 2ull * kHalfE * 4;              // [2][64] neighbour of each of this CTA's edges
        rpw = o;    o += (size_t)kTileE * 4;
        rho = o;    o += (size_t)kHalfE * kTcMaxRbf * 2;
        rrs = o;    o += (size_t)kHalfE * kTcMaxRbf * 4;
        wga = o;    o += (size_t)kTcMaxRbf * kMaxHeads * 4;
        o = (o + 1023) & ~size_t(1023);
        b2 = o;     o += 2ull * kB2Blocks * kB2Bytes;     // rotate-back operand blocks, two buffers
        slots = o;  o += (2 * kTileE + 8) * 4;            // node segments of the tile: start, node, count
        req = o;    o += 2 * ((2 * kB2Blocks + 4) * 4) + 16;  // per buffer: MMA requests, header, block parameters; mailbox
        o += 3 * 2 * kB2Blocks * 4 + 16;                      // first-pass lists per group kind (per tile), counts
        o = (o + 7) & ~size_t(7);
        bars = o;   o += (2 * kNS + 20) * 8;
        misc = o;   o += 64 + 4 * kHalfE * 4;  // TMEM base, abort flag, last slot; gate (i, j) lists
        dsub = o;   o += 16 * 8;
        total = o;
        (void)n_rbf;
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

// tcgen05.mma kind::f16 with the accumulate flag as an immediate (no predicate setup in the issue loop)
__device__ __forceinline__ void umma_f(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, int accumulate) {
    if (accumulate)
        asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, 1;" ::"r"(d), "l"(a), "l"(b), "r"(idesc)
                     : "memory");
    else
        asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, 0;" ::"r"(d), "l"(a), "l"(b), "r"(idesc)
                     : "memory");
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Rotate-back operand block: 16 rows (m') x 16 K (edges) fp16, no swizzle,
// K-major core matrices (8 rows x 16 bytes) 128 bytes apart along K and 256
// bytes apart along rows. Element (m', k) in halves:
__device__ __forceinline__ int b2_off(int mp, int k) { return ((mp >> 3) * 2 + (k >> 3)) * 64 + (mp & 7) * 8 + (k & 7); }
__device__ __forceinline__ uint64_t sdesc_b2(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(128u >> 4) << 16;   // leading byte offset: next core matrix along K
    d |= (uint64_t)(256u >> 4) << 32;   // stride byte offset: next 8-row group
    d |= (uint64_t)1u << 46;            // descriptor version (sm_100)
    return d;                           // swizzle: none
}
// kind::f16, D fp32, A and B fp16, K-major, M = 256 (a CTA pair), N = n, optional negation of A
__host__ __device__ constexpr uint32_t idesc_pair(int n, bool neg_a) {
    return (1u << 4) | ((neg_a ? 1u : 0u) << 13) | ((uint32_t)(n >> 3) << 17) | ((256u >> 4) << 24);
}

__device__ __forceinline__ void umma_ta(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, int accumulate) {
    if (accumulate)
        asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 1;" ::"r"(d), "r"(a_tmem), "l"(b),
                     "r"(idesc)
                     : "memory");
    else
        asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 0;" ::"r"(d), "r"(a_tmem), "l"(b),
                     "r"(idesc)
                     : "memory");
}

// TMEM column (within an accumulator's 128) of the fp16 operand of edges
// 16J..16J+15 after the in-place conversion (two fp16 per 32-bit column).
__device__ __forceinline__ int a2col(int J) { return 8 * J; }
// Rotate-back result regions (32 columns each, N of the pair MMA) inside a
// group's 256 columns: the halves of the two accumulators that the conversion
// has freed. In region k, CTA r's results are columns 16r..16r+15.
__device__ __forceinline__ int d2col(int k) { return 64 + 32 * (k & 1) + 128 * (k >> 1); }

// Wigner slice a CTA's accumulator needs: block (l3, mu) for the 128 edges of
// the pair tile, the first 64 from the even CTA's global copy and the rest
// from the odd CTA's (Dg0, Dg1). Queued on `bar` into `dst`; returns bytes.
__device__ __forceinline__ uint32_t stage_block(int l3, int mu, const __half2* Dg0, const __half2* Dg1, uint8_t* dst,
                                                uint64_t* bar) {
    const uint32_t half = (uint32_t)kHalfE * npair(l3) * 4;
    bulk_load(dst, Dg0 + dglob_block(l3, mu), half, bar);
    bulk_load(dst + half, Dg1 + dglob_block(l3, mu), half, bar);
    return 2 * half;
}


// Degree, channel and validity of this CTA's rows of accumulator a (a2 = 0) or b
// (a2 = 1, m = 0 groups) of group g for TMEM lane `row`: rows r0 + 128 rank + row of
// the group's block (o+/o- share the rows when mu > 0).
__device__ __forceinline__ void epi_rows(const TcGroup& g, int a2, int rank, int row, int L, int C, int& l3, int& c,
                                         bool& valid) {
    const int nrow = g.mu > 0 ? (L + 1 - g.mu) * C : (L + 1) * C;
    const int r0 = (a2 == 0 || g.mu > 0) ? g.row0 : g.row0b;
    const int rr = r0 + 128 * rank;
    valid = r0 >= 0 && rr < nrow;
    const int rc = valid ? rr + row : 0;
    l3 = (g.mu > 0 ? g.mu : 0) + (valid ? rr / C : 0);
    c = rc % C;
}

// Shared state of the epilogue's rotate-back passes (pointers into shared memory).
struct EpiShared {
    const int* sl_start;   // [segments + 1] first edge of each node segment, then the end
    uint32_t* req0;        // per buffer: requests [kB2Blocks], header [4], block parameters [kB2Blocks]
    uint8_t* b2s;          // operand blocks, two buffers
    const uint8_t* dstage; // staged Wigner slices, two buffers of dstride bytes
    size_t dstride;
};
__device__ __forceinline__ uint32_t* epi_req(const EpiShared& E, int q) { return E.req0 + q * (2 * kB2Blocks + 4); }
__device__ __forceinline__ int* epi_reqh(const EpiShared& E, int q) {
    return reinterpret_cast<int*>(E.req0 + q * (2 * kB2Blocks + 4) + kB2Blocks);
}
__device__ __forceinline__ uint32_t* epi_reqbp(const EpiShared& E, int q) {
    return E.req0 + q * (2 * kB2Blocks + 4) + kB2Blocks + 4;
}

// Request list of a rotate-back pass over segments [s0, s1) for a group kind: 0 =
// one m = 0 block (one accumulator), 1 = two m = 0 blocks (a, b), 2 = |m| >= 1
// (signs +, -). Entry: (result column, operand column, block, accumulate); block
// parameters: (segment, accumulator, 16-edge step). Returns the entry count.
__device__ __forceinline__ int epi_build_list(const int* sl_start, int kind, int s0, int s1, uint32_t* rl, uint32_t* bpl) {
    int n = 0;
    const int nacc = kind == 0 ? 1 : 2;
    for (int sg = s0; sg < s1; ++sg) {
        const int ea = sl_start[sg], eb = sl_start[sg + 1];
        for (int a2 = 0; a2 < nacc; ++a2) {
            const int dcol = kind == 1 ? d2col((sg - s0) + 2 * a2) : d2col(sg - s0);
            for (int J = ea >> 4; J <= (eb - 1) >> 4; ++J) {
                const bool first = (J == (ea >> 4)) && (a2 == 0 || kind != 2);
                rl[n] = (uint32_t)dcol | ((uint32_t)(128 * a2 + a2col(J)) << 8) | ((uint32_t)n << 16) |
                        ((first ? 0u : 1u) << 24);
                bpl[n] = (uint32_t)sg | ((uint32_t)a2 << 8) | ((uint32_t)J << 16);
                ++n;
            }
        }
    }
    return n;
}

// This CTA's operand blocks for a rotate-back pass of group gg (global group count
// gc2) from a request list (rl, bpl, n entries) into buffer gc2 & 1, and the
// buffer's header. Called by all epilogue threads; et = thread index, ew = warp.
// A warp takes blocks ew, ew + 4, ...: all their loads are issued before any is
// used.
constexpr int kBlkPerWarp = (kB2Blocks + kEpiThreads / 32 - 1) / (kEpiThreads / 32);
__device__ __forceinline__ void epi_prep_pass(const EpiShared& E, const TcGroup& gg, long long gc2, const uint32_t* rl,
                                              const uint32_t* bpl, int n, int rank, int L, int C, int et, int ew,
                                              int lane, long long* dt) {
    const long long t0 = dt ? clock64() : 0;
    const int q = (int)(gc2 & 1);
    int l3a, ca, l3b, cb2;
    bool va, vb;
    epi_rows(gg, 0, rank, 0, L, C, l3a, ca, va);
    epi_rows(gg, 1, rank, 0, L, C, l3b, cb2, vb);
    if (gg.mu > 0) { l3b = l3a; vb = va; }
    const bool tb = gg.mu == 0 && gg.row0b >= 0;
    if (et == 0) {
        epi_reqh(E, q)[0] = n;
        epi_reqh(E, q)[1] = q;  // TMEM slot of the group
        reinterpret_cast<const uint32_t**>(epi_reqh(E, q) + 2)[0] = rl;  // the list warp A issues
    }
    const long long t1 = dt ? clock64() : 0;
    const uint8_t* dsl = E.dstage + q * E.dstride;
    const int npa = npair(l3a);
    const int mp = lane & 15, kg = lane >> 4;
    const bool hi_sign = gg.mu > 0;
    long long tl = 0;
    for (int i0 = 0; i0 < kBlkPerWarp; i0 += 3) {  // three blocks in flight at a time
        uint4 pr[3][2];
        int eaa[3], ebb[3], e0a[3];
        bool hia[3];
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const int k = ew + (i0 + i) * (kEpiThreads / 32);
            pr[i][0] = make_uint4(0, 0, 0, 0);
            pr[i][1] = make_uint4(0, 0, 0, 0);
            eaa[i] = 0; ebb[i] = 0; e0a[i] = 0; hia[i] = false;
            if (k < n) {
                const uint32_t bp = bpl[k];
                const int sg = bp & 255, a2 = (bp >> 8) & 255, J = bp >> 16;
                eaa[i] = E.sl_start[sg];
                ebb[i] = E.sl_start[sg + 1];
                const int l3 = a2 == 0 ? l3a : l3b;
                const bool vv = a2 == 0 ? va : vb;
                const int NP = npair(l3);
                const __half2* Dq = reinterpret_cast<const __half2*>(dsl) + ((tb && a2 == 1) ? kTileE * npa : 0);
                hia[i] = hi_sign && a2 == 1;  // sign -: the pair's high half
                const int e0 = 16 * J + 8 * kg;  // this lane's 8 edges (one half of the pair tile)
                e0a[i] = e0;
                if (vv && mp < 2 * l3 + 1) {
                    const uint4* src = reinterpret_cast<const uint4*>(Dq + ((e0 >> 6) * NP + mp) * kHalfE + (e0 & 63));
                    pr[i][0] = src[0];
                    pr[i][1] = src[1];
                }
            }
        }
        if (dt) tl -= clock64();
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const int k = ew + (i0 + i) * (kEpiThreads / 32);
            if (k < n) {
                const __half2* ph = reinterpret_cast<const __half2*>(pr[i]);
                uint32_t pk[4];
#pragma unroll
                for (int i2 = 0; i2 < 4; ++i2) {
                    float f2[2];
#pragma unroll
                    for (int i1 = 0; i1 < 2; ++i1) {
                        const int e = e0a[i] + 2 * i2 + i1;
                        const __half2 pv = ph[2 * i2 + i1];
                        f2[i1] = (e >= eaa[i] && e < ebb[i]) ? __half2float(hia[i] ? __high2half(pv) : __low2half(pv)) : 0.f;
                    }
                    pk[i2] = pack_h2(f2[0], f2[1]);
                }
                *reinterpret_cast<uint4*>(E.b2s + (size_t)q * kB2Blocks * kB2Bytes + (size_t)k * kB2Bytes +
                                          2 * b2_off(mp, 8 * kg)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        }
        if (dt) tl += clock64();
    }
    const long long t2 = dt ? clock64() - tl : 0;  // (loads and stores are timed together below)
    const long long t3 = dt ? clock64() : 0;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // blocks -> tensor core
    if (dt) {
        const long long t4 = clock64();
        dt[0] += t1 - t0; dt[1] += t2 - t1; dt[2] += t3 - t2; dt[3] += t4 - t3;
    }
}

// 16 accumulator columns of chunk j (edges 16j..16j+15) -> fp16 p o, packed into
// 8 columns in place (p = softmax weights of the row's head, 16 floats)
__device__ __forceinline__ void epi_convert16(uint32_t taddr_acc, const float* v, const float* p16, int j) {
    const float4* p4 = reinterpret_cast<const float4*>(p16);
    uint32_t u[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float4 pa = p4[k];
        u[2 * k] = pack_h2(v[4 * k] * pa.x, v[4 * k + 1] * pa.y);
        u[2 * k + 1] = pack_h2(v[4 * k + 2] * pa.z, v[4 * k + 3] * pa.w);
    }
    tmem_st8(taddr_acc + a2col(j), u);
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
    float* php = reinterpret_cast<float*>(smem + S.php);  // [2][H][128] softmax weight per head and edge
    int* nid = reinterpret_cast<int*>(smem + S.nid);      // [2][128]
    int* jn = reinterpret_cast<int*>(smem + S.jn);        // [2][64]
    uint8_t* b2s = smem + S.b2;                                   // rotate-back operand blocks
    int* sl_start = reinterpret_cast<int*>(smem + S.slots);       // [129] first edge of each node segment
    int* sl_node = sl_start + kTileE + 1;                         // [128] its node
    int* sl_count = sl_node + kTileE;                             // number of segments
    // per buffer q: req(q)[kB2Blocks] MMA requests, reqh(q)[4] count and TMEM slot,
    // reqbp(q)[kB2Blocks] block parameters; mailbox: buffer of the pass being handed over
    uint32_t* req0 = reinterpret_cast<uint32_t*>(smem + S.req);
    auto req = [=](int q) { return req0 + q * (2 * kB2Blocks + 4); };
    auto reqh = [=](int q) { return reinterpret_cast<int*>(req0 + q * (2 * kB2Blocks + 4) + kB2Blocks); };
    auto reqbp = [=](int q) { return req0 + q * (2 * kB2Blocks + 4) + kB2Blocks + 4; };
    volatile int* mailbox = reinterpret_cast<volatile int*>(req0 + 2 * (2 * kB2Blocks + 4));
    // first-pass request lists of the current tile per group kind (0: one m = 0 block, 1: two
    // m = 0 blocks, 2: |m| >= 1): entries [kB2Blocks], block parameters [kB2Blocks]; counts
    uint32_t* klist = req0 + 2 * (2 * kB2Blocks + 4) + 4;
    int* klistn = reinterpret_cast<int*>(klist + 3 * 2 * kB2Blocks);
    int* rpw = reinterpret_cast<int*>(smem + S.rpw);
    __half* rho = reinterpret_cast<__half*>(smem + S.rho);  // [64][16] radial basis, fp16 (gate warps)
    float* rrs = reinterpret_cast<float*>(smem + S.rrs);    // [64][16] radial basis, fp32 (logits)
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S.bars);
    uint64_t* full = bars;            // stage landed in both CTAs (even CTA's barrier; TMA transactions)
    uint64_t* empty = bars + kNS;     // stage consumed (both MMA warps of the even CTA, to both CTAs)
    uint64_t* tfull = bars + 2 * kNS; // accumulator slot complete (both MMA warps, to both CTAs)
    uint64_t* tempty = tfull + 2;     // accumulator slot drained (even CTA's barrier; both epilogues)
    uint64_t* xready = tempty + 2;    // tile buffer produced (both producers, to both CTAs)
    uint64_t* xfree = xready + 2;     // tile buffer consumed (both epilogues, to both CTAs)
    uint64_t* dbar = xfree + 2;       // epilogue Wigner staging, per buffer
    uint64_t* fin = dbar + 2;         // [2] final commits of the two MMA warps
    uint64_t* gfull = fin + 2;        // value gate of a tile buffer written (gate warps -> producer)
    uint64_t* gempty = gfull + 2;     // value gate of a tile buffer consumed (producer -> gate warps)
    uint64_t* jfull = gempty + 2;     // fused traversal: (i, j) of a tile buffer listed (gate warps -> producer)
    uint64_t* d2full = jfull + 2;     // rotate-back MMAs of a pass complete (to both CTAs)
    uint64_t* a2ready = d2full + 1;   // rotate-back operands of a pass ready (even CTA's barrier; both epilogues)
    uint32_t* tmem_sm = reinterpret_cast<uint32_t*>(smem + S.misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S.misc + 8);
    int* last_slot = reinterpret_cast<int*>(smem + S.misc + 16);  // producer: node slot of the last edge
    int* gij = reinterpret_cast<int*>(smem + S.misc + 64);        // gate warps: [2][2][64] (i, j) per edge
    long long* dsub = reinterpret_cast<long long*>(smem + S.dsub);  // sub-step cycle sums (timers on)
    float* wga = reinterpret_cast<float*>(smem + S.wga);            // [16][H] logit-gate weights
    const bool dbgon = P.dbg != nullptr;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();      // 0: issues the pair's MMAs
    const uint32_t peer = rank ^ 1u;
    const int pair = blockIdx.x >> 1;
    // cluster addresses of barriers in the peer / even CTA
    auto at_peer = [=](const void* local) { return mapa(smem_u32(local), peer); };
    auto at_even = [=](const void* local) { return mapa(smem_u32(local), 0u); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNS; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 2); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + b, 2);
            mbar_init(tempty + b, 2 * kEpiThreads);
            mbar_init(xready + b, 2 * 128);
            mbar_init(xfree + b, 2 * kEpiThreads);
            mbar_init(dbar + b, 1);
        }
        mbar_init(fin, 1);
        mbar_init(fin + 1, 1);
        mbar_init(d2full, 1);
        mbar_init(a2ready, 2 * kEpiThreads);
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
        tmem_alloc2(tmem_sm, 512);
        tmem_relinquish2();
    }
    tc_fence_before();
    cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
    tc_fence_after();
    const uint32_t tmem = *tmem_sm;

    const int n_begin = P.part[pair], n_end = P.part[pair + 1];
    const int e_begin = P.row_ptr[n_begin], e_end = P.row_ptr[n_end];
    const int ntiles = (e_end - e_begin + kTileE - 1) / kTileE;
    const int ng = P.n_groups;
    const int eoff = (int)rank * kHalfE;  // this CTA's edges within a pair tile

    if (warp >= 4 && warp < 8) {
        // ---------------- producer ----------------
        const int p = threadIdx.x - 128;
        const float inv_sqrt_dh = rsqrtf((float)dh);
        const float inv_s = P.scale[1];
        const int CG = C / 8;
        const int Gv = (L + 1) * C;
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
            // both epilogues are done with this buffer (this producer also writes the peer's copy)
            const bool okw = (t < 2) || wait_cluster(xfree + b, ((t - 2) >> 1) & 1, abort_flag, P.status, w_free);
            if (!bar_and(1, 128, okw)) break;
            const long long c_a = clock64();
            const int e0 = e_begin + t * kTileE + eoff;       // this CTA's first edge
            const int ne = max(0, min(kHalfE, e_end - e0));   // and count
            // window of row_ptr after the node of this CTA's first edge
            {
                int nb0;
                if (t == 0) {
                    const int ef = min(e0, max(e_begin, e_end - 1));
                    int lo = n_begin, hi = n_end - 1;
                    while (lo < hi) {
                        int mid = (lo + hi + 1) >> 1;
                        if (P.row_ptr[mid] <= ef) lo = mid; else hi = mid - 1;
                    }
                    nb0 = lo;
                } else {
                    nb0 = *last_slot;  // node slot of this CTA's last edge of the previous tile
                }
                nbase = nb0;
                const int n = nbase + 1 + p;
                rpw[p] = (n <= n_end) ? P.row_ptr[n] : 0x7fffffff;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (P.cells) {
                // fused traversal: the gate warps list (atom, neighbour) of this CTA's edges in
                // gij[b]; they refill it only after gempty[b], i.e. after this tile's P2
                const bool okj = wait_t(jfull + b, (t >> 1) & 1, abort_flag, P.status, w_free);
                if (!bar_and(1, 128, okj)) break;
            }
            tlast = c_a;
            E2F_TICK(0);
            __half2* Dg = P.dscr + (size_t)(blockIdx.x * 2 + b) * dglob_pairs();
            // P1: one edge per thread: frame, Wigner pairs (fp16x2; shared copy for
            // the rotation below, global copy for the epilogues of both CTAs)
            if (p < kHalfE) {
                __half2* Dh = dph + (size_t)p * DPS;
                const uint32_t nid_peer = at_peer(nid + b * kTileE + eoff + p);
                if (p < ne) {
                    const int e = e0 + p;
                    const int* gl = gij + b * 2 * kHalfE;  // fused traversal: [i x 64][j x 64]
                    const int j = P.cells ? gl[kHalfE + p] : P.col[e];
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
                    if (p == ne - 1) *last_slot = i;
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
                            uint32_t* gq = reinterpret_cast<uint32_t*>(Dg + dglob_block(l, mu)) + p;
#pragma unroll
                            for (int n4 = 0; n4 < npair(l); n4 += 4) {
                                uint32_t wv[4];
#pragma unroll
                                for (int t4 = 0; t4 < 4; ++t4) {
                                    const int n = n4 + t4;
                                    const float a0 = n < w ? Dl[(l + mu) * w + n] : 0.f;
                                    const float b0 = n < w ? Dl[(l - mu) * w + n] : 0.f;
                                    wv[t4] = pack_h2(a0, b0);
                                    gq[(size_t)n * kHalfE] = wv[t4];  // a warp writes 32 consecutive words
                                }
                                sq[n4 / 4] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
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
                    nid[b * kTileE + eoff + p] = i;
                    st_cluster_u32(nid_peer, (uint32_t)i);
                    jn[b * kHalfE + p] = j;
                } else {
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int l = 0; l <= L; ++l)
#pragma unroll
                        for (int mu = 0; mu <= l; ++mu) {
                            uint32_t* gq = reinterpret_cast<uint32_t*>(Dg + dglob_block(l, mu)) + p;
                            for (int n = 0; n < npair(l); ++n) gq[(size_t)n * kHalfE] = 0u;
                        }
                    for (int a = 0; a < DPS; a += 4) *reinterpret_cast<uint4*>(Dh + a) = z;
                    for (int h = 0; h < H; ++h) {
                        php[(b * H + h) * kTileE + eoff + p] = 0.f;
                        st_cluster_f32(at_peer(php + (b * H + h) * kTileE + eoff + p), 0.f);
                    }
                    nid[b * kTileE + eoff + p] = -1;
                    st_cluster_u32(nid_peer, 0xffffffffu);
                    jn[b * kHalfE + p] = 0;
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            E2F_TICK(6);
            // logits and softmax weights, one (edge, head) pair per thread and step: the
            // thread's head h = p % H is fixed (H divides 128), the H lanes of an edge read
            // its key row as consecutive float4; written to both CTAs
            {
                const int h = p % H, d4 = dh / 4;
                float wh[kTcMaxRbf];
#pragma unroll
                for (int kb = 0; kb < kTcMaxRbf; ++kb) wh[kb] = wga[kb * H + h];
#pragma unroll 2
                for (int e = p / H; e < ne; e += 128 / H) {
                    const int i = nid[b * kTileE + eoff + e], j = jn[b * kHalfE + e];
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
                    php[(b * H + h) * kTileE + eoff + e] = pw;
                    st_cluster_f32(at_peer(php + (b * H + h) * kTileE + eoff + e), pw);
                }
            }
            E2F_TICK(5);
            asm volatile("bar.sync 1, 128;" ::: "memory");
            E2F_TICK(7);
            const long long c_b = clock64();
            c_p1 += c_b - c_a;
            // P2: rotated, gated features -> scratch row (e), all |m| blocks (fp16, packed math)
            {
                const bool okg = wait_t(gfull + b, (t >> 1) & 1, abort_flag, P.status, w_free);
                if (!bar_and(1, 128, okg)) break;
            }
            const __half* gs = P.gscr + ((size_t)blockIdx.x * 2 + b) * kHalfE * Gv;
            __half* xrow0 = P.xs + ((size_t)(blockIdx.x * 2 + b) * kHalfE) * KT;
            for (int it = p; it < kHalfE * CG; it += 128) {
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
                const int j = jn[b * kHalfE + e];
                if (c0 == 0 && e + 8 < ne)  // neighbour row of the edge one round ahead
                    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                                     P.x + (size_t)jn[b * kHalfE + e + 8] * KT),
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
            // generic-proxy stores (features, Wigner pairs) -> visible to TMA / bulk copies; the
            // shared-memory stores into the peer (nid, php) are released by the cluster arrive
            asm volatile("fence.proxy.async.global;" ::: "memory");
            mbar_arrive(xready + b);
            mbar_arrive_cluster(at_peer(xready + b));
            c_p2 += clock64() - c_b;
        }
        if (P.dbg && p == 0) {
            long long* d = P.dbg + blockIdx.x * kDbgSlots;
            d[0] = w_free; d[1] = clock64() - c_start; d[11] = c_p1; d[12] = c_p2;
            for (int k = 0; k < 8; ++k) d[14 + k] = dsub[k];
        }
#undef E2F_TICK
    } else if (warp == 12) {
        // ---------------- TMA (both CTAs) ----------------
        // Each CTA loads its 128 weight rows and its 64 edges of the feature tile into
        // its own ring; every load's completion is counted on the even CTA's `full`
        // barrier, where the even CTA expects the bytes of both.
        if (lane == 0) {
            const uint64_t pol_xs = policy_evict_last();
            int stage = 0;
            uint32_t ph = 0;
            bool ok = true;
            int pending[kNS];
            for (int s2 = 0; s2 < kNS; ++s2) pending[s2] = -1;
            long long w_x = 0, w_e = 0;
            const long long c_start = clock64();
            (void)pol_xs;
            for (int t = 0; t < ntiles && ok; ++t) {
                const int b = t & 1;
                if (!wait_cluster(xready + b, (t >> 1) & 1, abort_flag, P.status, w_x)) { ok = false; break; }
                const int rowT = (blockIdx.x * 2 + b) * kHalfE;
                for (int gi = 0; gi < ng && ok; ++gi) {
                    const TcGroup g = P.groups[gi];
                    const int wr0 = g.row0 + 128 * (int)rank, wr0b = g.row0b + 128 * (int)rank;
                    const int ntw = g.mu > 0 ? 2 : (g.row0b >= 0 ? 2 : 1);
                    const int ntx = g.mu > 0 ? 2 : 1;
                    const uint32_t bytes_cta = (uint32_t)(ntw * kWSlot + ntx * kXSlot);
                    for (int kk = 0; kk < g.klen; kk += kKS) {
                        if (!wait_t(empty + stage, ph ^ 1, abort_flag, P.status, w_e)) { ok = false; break; }
                        uint8_t* st = ring + (size_t)stage * kStage;
                        const uint32_t fb = at_even(full + stage);
                        // local barrier, local waiters: a CTA-scope arrive (a cluster-scope release
                        // here would wait for this thread's loads in flight)
                        if (rank == 0) mbar_arrive_tx(full + stage, 2 * bytes_cta);
                        if (g.mu > 0) {
                            tma_load_2d_pair(st, &T.w[g.wa], kk, wr0, fb);
                            tma_load_2d_pair(st + kWSlot, &T.w[g.wb], kk, wr0, fb);
                            tma_load_2d_pair(st + 2 * kWSlot, &T.xs, g.xoff0 + kk, rowT, fb);
                            tma_load_2d_pair(st + 2 * kWSlot + kXSlot, &T.xs, g.xoff1 + kk, rowT, fb);
                        } else {
                            tma_load_2d_pair(st, &T.w[g.wa], kk, wr0, fb);
                            if (g.row0b >= 0) tma_load_2d_pair(st + kWSlot, &T.w[g.wa], kk, wr0b, fb);
                            tma_load_2d_pair(st + 2 * kWSlot, &T.xs, g.xoff0 + kk, rowT, fb);
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
            // the loads this CTA issued complete before it can leave: the last use of each
            // stage is released (consumed) by the MMAs only after its data landed
            for (int s2 = 0; s2 < kNS; ++s2) {
                if (pending[s2] < 0) continue;
                const uint64_t t0 = gtimer();
                while (!mbar_try(empty + s2, (uint32_t)pending[s2]) && gtimer() - t0 < kWaitNs) {
                }
            }
        }
        __syncwarp();
    } else if (rank == 0 && (warp == 13 || warp == 8)) {
        // ---------------- MMA (even CTA; two issuing warps) ----------------
        // One M256 x N128 x K16 instruction covers both CTAs: rows 0-127 of the group's
        // weights and its accumulator lanes in the even CTA, rows 128-255 in the odd
        // one; the 128 edge columns come 64 from each CTA's feature tile. The issuing
        // thread runs in step with the tensor pipe, so two warps issue: A (warp 13) the
        // first accumulator of each group (o+, or the first m = 0 block), B (warp 8) the
        // second (o-, or the second block). Warp A also issues the rotate-back MMAs of
        // the previous group halfway through each group, in its own stream.
        const bool wa = warp == 13;
        if (lane == 0) {
            int stage = 0;
            uint32_t ph = 0;
            long long gcount = 0;
            bool ok = true;
            long long w_t = 0, w_f = 0;
            const long long c_start = clock64();
            constexpr uint32_t ID = idesc_pair(128, false), IDN = idesc_pair(128, true), ID2 = idesc_pair(32, false);
            // Operand descriptors of the ring stages, built once: the issue loop only
            // adds constant offsets (the start address field counts 16-byte units,
            // and every stage lies below 256 KB, so the additions never carry).
            const uint64_t dbase0 = sdesc_sw64(smem_u32(ring));
            constexpr uint64_t kWs = kWSlot >> 4, kXs = kXSlot >> 4, kKs = 32 >> 4, kSt = kStage >> 4;
            const uint64_t b2base = sdesc_b2(smem_u32(b2s));
            long long m_issue = 0, m_commit = 0, m_serv = 0;
            uint32_t a2ph = 0;
            // A rotate-back pass (its arrival on a2ready observed): the epilogues' request
            // list, identical in both CTAs, read from this one; passes arrive in order and
            // are issued in that order. Written as a macro, not a lambda, so that the loop
            // counters stay in registers.
#define E2F_ISSUE_PASS()                                                                                     \
    do {                                                                                                    \
        a2ph ^= 1;                                                                                          \
        tc_fence_after();                                                                                   \
        const int q_ = *mailbox;                                                                            \
        const int n_ = reqh(q_)[0];                                                                         \
        const uint32_t cbt_ = tmem + (uint32_t)reqh(q_)[1] * 256u;                                          \
        const uint32_t* rl_ = reinterpret_cast<const uint32_t* const*>(reqh(q_) + 2)[0];                    \
        const uint64_t bq_ = b2base + (uint64_t)q_ * (kB2Blocks * kB2Bytes >> 4);                           \
        for (int k_ = 0; k_ < n_; ++k_) {                                                                   \
            const uint32_t rq_ = rl_[k_];                                                                   \
            umma2_ts(cbt_ + (rq_ & 255u), cbt_ + ((rq_ >> 8) & 255u),                                       \
                     bq_ + (uint64_t)((rq_ >> 16) & 255u) * (kB2Bytes >> 4), ID2, (int)(rq_ >> 24));        \
        }                                                                                                   \
        umma2_commit_both(d2full);                                                                          \
    } while (0)
            // bounded wait that serves rotate-back passes arriving meanwhile; sets `ok`
#define E2F_WAIT_S(bar_, par_, acc_)                                                                         \
    do {                                                                                                    \
        if (!mbar_try((bar_), (par_))) {                                                                    \
            const long long c0_ = clock64();                                                                \
            const uint64_t t0_ = gtimer();                                                                  \
            while (!mbar_try((bar_), (par_))) {                                                             \
                if (wa && mbar_test(a2ready, a2ph)) E2F_ISSUE_PASS();                                        \
                if (*abort_flag) { ok = false; break; }                                                     \
                if (gtimer() - t0_ > kWaitNs) {                                                             \
                    *abort_flag = 1;                                                                        \
                    atomicExch(P.status, (int)E2F_ERR_TIMEOUT);                                             \
                    ok = false;                                                                             \
                    break;                                                                                  \
                }                                                                                           \
            }                                                                                               \
            (acc_) += clock64() - c0_;                                                                      \
        }                                                                                                   \
    } while (0)
            for (int t = 0; t < ntiles && ok; ++t) {
                for (int gi = 0; gi < ng && ok; ++gi, ++gcount) {
                    const TcGroup g = P.groups[gi];
                    const int slot = (int)(gcount & 1);
                    const uint32_t use = (uint32_t)(gcount >> 1);
                    E2F_WAIT_S(tempty + slot, (use & 1) ^ 1, w_t);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t d0 = tmem + slot * 256, d1 = d0 + 128;
                    const int kind = g.mu > 0 ? 2 : (g.row0b >= 0 ? 1 : 0);
                    for (int kk = 0; kk < g.klen; kk += kKS) {
                        E2F_WAIT_S(full + stage, ph, w_f);
                        if (!ok) break;
                        tc_fence_after();
                        const long long c_i0 = dbgon ? clock64() : 0;
                        // stage: weights A (0), B (kWs) / second block; features x+ (2 kWs), x- (+kXs)
                        const uint64_t a0 = dbase0 + (uint64_t)stage * kSt, a1 = a0 + kWs, x0 = a0 + 2 * kWs,
                                       x1 = x0 + kXs;
                        if (kind == 2) {
                            if (wa) {  // o+ = A h+ - B h-
                                if (kk == 0) umma2_ss(d0, a0, x0, ID, 0); else umma2_ss(d0, a0, x0, ID, 1);
                                umma2_ss(d0, a1, x1, IDN, 1);
                                umma2_ss(d0, a0 + kKs, x0 + kKs, ID, 1);
                                umma2_ss(d0, a1 + kKs, x1 + kKs, IDN, 1);
                            } else {   // o- = B h+ + A h-
                                if (kk == 0) umma2_ss(d1, a1, x0, ID, 0); else umma2_ss(d1, a1, x0, ID, 1);
                                umma2_ss(d1, a0, x1, ID, 1);
                                umma2_ss(d1, a1 + kKs, x0 + kKs, ID, 1);
                                umma2_ss(d1, a0 + kKs, x1 + kKs, ID, 1);
                            }
                        } else if (wa) {
                            if (kk == 0) umma2_ss(d0, a0, x0, ID, 0); else umma2_ss(d0, a0, x0, ID, 1);
                            umma2_ss(d0, a0 + kKs, x0 + kKs, ID, 1);
                        } else if (kind == 1) {
                            if (kk == 0) umma2_ss(d1, a1, x0, ID, 0); else umma2_ss(d1, a1, x0, ID, 1);
                            umma2_ss(d1, a1 + kKs, x0 + kKs, ID, 1);
                        }
                        const long long c_i1 = dbgon ? clock64() : 0;
                        umma2_commit_both(empty + stage);
                        if (++stage == kNS) { stage = 0; ph ^= 1; }
                        if (dbgon) {
                            const long long c_i2 = clock64();
                            m_issue += c_i1 - c_i0; m_commit += c_i2 - c_i1;
                        }
                        // a rotate-back pass of the previous group, if its operands are ready
                        // (while this warp polls, the other warp's MMAs keep the pipe busy)
                        if (wa && mbar_test(a2ready, a2ph)) {
                            const long long c_s0 = dbgon ? clock64() : 0;
                            E2F_ISSUE_PASS();
                            if (dbgon) m_serv += clock64() - c_s0;
                        }
                    }
                    if (ok) umma2_commit_both(tfull + slot);
                }
            }
            // further passes of the last groups: serve them until both slots are released
            if (wa) {
                for (int s2 = 0; s2 < 2 && ok; ++s2) {
                    const long long nuse = (gcount + 1 - s2) / 2;  // uses of slot s2
                    if (nuse > 0) E2F_WAIT_S(tempty + s2, (uint32_t)((nuse & 1) ^ 1), w_t);
                }
            }
#undef E2F_WAIT_S
#undef E2F_ISSUE_PASS
            if (P.dbg && wa) {
                long long* d = P.dbg + blockIdx.x * kDbgSlots;
                d[5] = w_t; d[6] = w_f; d[7] = clock64() - c_start;
                d[25] = m_issue; d[26] = m_commit; d[27] = m_serv;
            }
            // every issued MMA completes (bounded wait) before TMEM is released
            uint64_t* fb = fin + (wa ? 0 : 1);
            umma2_commit_both(fb);
            const uint64_t t0 = gtimer();
            while (!mbar_try(fb, 0) && gtimer() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else if (warp >= 14) {
        // ---------------- value gate (warps 14-15), up to two tiles ahead ----------------
        // g[e][n] = rho(d_e) . W_rad[:, n] for this CTA's 64 edges of a tile and
        // n < (L+1)C, into a per-CTA global buffer per tile parity that the
        // producer's rotation reads.
        const int gp = threadIdx.x - 448, gw = warp - 14, g8 = lane >> 2, t4 = lane & 3;
        const int Gv = (L + 1) * C;
        long long w_g = 0;
        const long long c_start = clock64();
        for (int t = 0; t < ntiles; ++t) {
            const int b = t & 1;
            const bool okw = (t < 2) || wait_t(gempty + b, ((t - 2) >> 1) & 1, abort_flag, P.status, w_g);
            if (!bar_and(3, 64, okw)) break;
            const int e0 = e_begin + t * kTileE + eoff;
            const int ne = max(0, min(kHalfE, e_end - e0));
            int* gi = gij + b * 2 * kHalfE;
            if (P.cells) {  // fused traversal: (atom, neighbour) of each edge from the cell lists
                auto slot_of = [&](int e) {
                    int lo = n_begin, hi = n_end - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (P.row_ptr[mid] <= e) lo = mid; else hi = mid - 1;
                    }
                    return lo;
                };
                if (ne > 0) {
                    const int s_first = slot_of(e0), s_last = slot_of(e0 + ne - 1);
                    for (int sl = s_first + (warp - 14); sl <= s_last; sl += 2) {
                        const int base = P.row_ptr[sl], ia = P.cv.sidx[sl];
                        warp_neighbors(
                            P.cv, P.cv.spos[sl], ia,
                            [&](int k, int j) {
                                const int e = base + k;
                                if (e >= e0 && e < e0 + ne) {
                                    gi[e - e0] = ia;
                                    gi[kHalfE + e - e0] = j;
                                }
                            },
                            0, sl);
                    }
                }
                asm volatile("bar.sync 3, 64;" ::: "memory");
                mbar_arrive(jfull + b);  // releases the lists to the producer (CTA scope)
            }
            {  // radial basis of this CTA's edges, one per thread
                const int k = gp;
                float rr[kTcMaxRbf];
                if (k < ne) {
                    const int e = e0 + k;
                    int lo, j;
                    if (P.cells) {
                        lo = gi[k];
                        j = gi[kHalfE + k];
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
            // one k = 16 mma.sync per 16 edges x 8 columns; warp gw takes edge blocks 2 gw, 2 gw + 1
            __half* gs = P.gscr + ((size_t)blockIdx.x * 2 + b) * kHalfE * Gv;
            uint32_t af[2][4];
#pragma unroll
            for (int mb = 0; mb < 2; ++mb) {
                const __half* rr0 = rho + ((2 * gw + mb) * 16 + g8) * kTcMaxRbf + 2 * t4;
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
                for (int mb = 0; mb < 2; ++mb) {
                    float acc4[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_16816(acc4, af[mb], bf);
                    const int e = (2 * gw + mb) * 16 + g8;
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
    } else if (warp < 4) {
        // ---------------- epilogue (warps 0-3, both CTAs) ----------------
        // Per group, the rotate-back v = D(R)^T o weighted by the softmax and summed
        // over each node's edges runs on the tensor cores:
        //   1. conversion: each thread owns one TMEM lane (one output row (l3, c) of
        //      this CTA's half of the group) and converts its 128 edge columns to
        //      fp16 p_e o[c, e] in place (packed into the accumulator's first 64 columns);
        //   2. per pass over up to 4 node segments of the tile (2 for a two-block m = 0
        //      group), each CTA builds 16-row operand blocks B2[m'][e] = D_e^{l3}[+-mu][m']
        //      (zero outside the node's edges) for its own degree l3, and the even CTA's
        //      MMA warp A issues M256 N32 K16 pair MMAs D2[c][n] += sum_e A2[c][e] B2[n][e]
        //      (A2 = the converted operand in TMEM); for a lane of CTA r the columns
        //      16r..16r+15 of a node's 32 are its own degree's rotate-back;
        //   3. drain: out[node][l3, m'][c] += D2[c][16r + m'] (m' < 2 l3 + 1), each output
        //      element added by one thread (lane c of the CTA holding row (l3, c)) in
        //      program order, so the order of additions is fixed.
        // Every decision to stop goes through bar_and, so the 128 threads leave
        // together and no thread is left at a named barrier.
        const int r = threadIdx.x;
        const int row = r;                               // this thread's TMEM lane
        const int et = r;
        const int ew = warp;                             // epilogue warp 0..3
        const uint32_t tlane = tmem + ((uint32_t)(32 * warp) << 16);
        long long gcount = 0;
        bool ok = true;
        long long w_x = 0, w_t = 0;
        long long staged[2] = {-1, -1};  // last group index staged into each buffer (thread 0)
        uint32_t d2ph = 0;
        const long long c_start = clock64();
        EpiShared E;
        E.sl_start = sl_start;
        E.req0 = req0;
        E.b2s = b2s;
        E.dstage = dstage;
        E.dstride = S.dstride;
        const __half2* dg_even = P.dscr + (size_t)((blockIdx.x & ~1) * 2) * dglob_pairs();
        const __half2* dg_odd = P.dscr + (size_t)((blockIdx.x | 1) * 2) * dglob_pairs();
        // stages the Wigner slices of a group's accumulators in this CTA (one thread)
#define E2F_STAGE_GROUP(gg_, b_, dst_, bar_)                                                                 \
    do {                                                                                                    \
        const TcGroup gq_ = (gg_);                                                                          \
        const __half2* Dg0_ = dg_even + (size_t)(b_) * dglob_pairs();                                       \
        const __half2* Dg1_ = dg_odd + (size_t)(b_) * dglob_pairs();                                        \
        int l3a_, ca_, l3b_, cb_;                                                                           \
        bool va_, vb_;                                                                                      \
        epi_rows(gq_, 0, (int)rank, 0, L, C, l3a_, ca_, va_);                                               \
        epi_rows(gq_, 1, (int)rank, 0, L, C, l3b_, cb_, vb_);                                               \
        const bool tb_ = gq_.mu == 0 && gq_.row0b >= 0;                                                     \
        const uint32_t ba_ = (uint32_t)kTileE * npair(l3a_) * 4;                                            \
        const uint32_t bb_ = tb_ ? (uint32_t)kTileE * npair(l3b_) * 4 : 0u;                                 \
        mbar_arrive_tx((bar_), ba_ + bb_);                                                                  \
        stage_block(l3a_, gq_.mu, Dg0_, Dg1_, (dst_), (bar_));                                              \
        if (tb_) stage_block(l3b_, 0, Dg0_, Dg1_, (dst_) + ba_, (bar_));                                    \
    } while (0)
        for (int t = 0; t < ntiles; ++t) {
            const int b = t & 1;
            const bool okx = wait_cluster(xready + b, (t >> 1) & 1, abort_flag, P.status, w_x);
            if (!bar_and(2, kEpiThreads, ok && okx)) { ok = false; break; }
            const int* nb = nid + b * kTileE;
            if (r == 0) {
                E2F_STAGE_GROUP(P.groups[0], b, dstage + (gcount & 1) * S.dstride, dbar + (gcount & 1));
                staged[gcount & 1] = gcount;
            }
            // node segments of the tile (its edges are the prefix with nid >= 0)
            if (ew == 0) {
                int f[4], c = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int e = 4 * lane + k;
                    f[k] = nb[e] >= 0 && (e == 0 || nb[e] != nb[e - 1]);
                    c += f[k];
                }
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += v;
                }
                int pos = incl - c;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int e = 4 * lane + k;
                    if (f[k]) { sl_start[pos] = e; sl_node[pos] = nb[e]; ++pos; }
                }
                // end of the last segment: the first padding edge (or 128)
                int ne_l = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) ne_l += nb[4 * lane + k] >= 0;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ne_l += __shfl_xor_sync(0xffffffffu, ne_l, o);
                const int ns = __shfl_sync(0xffffffffu, incl, 31);
                if (lane == 0) { sl_count[0] = ns; sl_start[ns] = ne_l; }
                __syncwarp();
                if (lane < 3) {  // first-pass lists per group kind, one lane each
                    const int per = lane == 1 ? 2 : 4;
                    uint32_t* kl = klist + lane * 2 * kB2Blocks;
                    klistn[lane] = epi_build_list(sl_start, lane, 0, min(ns, per), kl, kl + kB2Blocks);
                }
            }
            bool prepped = false;  // the current group's first pass was prepared during the previous group
            for (int gi = 0; gi < ng; ++gi, ++gcount) {
                // all threads are done with group gcount-1, so its staging buffer can be refilled
                if (!bar_and(2, kEpiThreads, ok)) { ok = false; break; }
                if (r == 0 && gi + 1 < ng) {
                    E2F_STAGE_GROUP(P.groups[gi + 1], b, dstage + ((gcount + 1) & 1) * S.dstride, dbar + ((gcount + 1) & 1));
                    staged[(gcount + 1) & 1] = gcount + 1;
                }
                const TcGroup g = P.groups[gi];
                const int slot = (int)(gcount & 1);
                const uint32_t use = (uint32_t)(gcount >> 1);
                const long long c_e0 = clock64();
                const uint32_t cb = (uint32_t)slot * 256u;
                const bool two = g.mu > 0 || g.row0b >= 0;
                int l3A, cA, l3B, cB;
                bool vA, vB;
                epi_rows(g, 0, (int)rank, row, L, C, l3A, cA, vA);
                epi_rows(g, 1, (int)rank, row, L, C, l3B, cB, vB);
                if (g.mu > 0) { l3B = l3A; cB = cA; vB = vA; }
                const int nseg = sl_count[0];
                const bool twob = g.mu == 0 && g.row0b >= 0;
                const int per = twob ? 2 : 4;  // segments per pass (result regions)
                if (!prepped) {
                    const bool okd = wait_t(dbar + slot, use & 1, abort_flag, P.status, w_t);
                    if (!bar_and(2, kEpiThreads, okd)) {
                        ok = false;
                        break;
                    }
                    const int kd = g.mu > 0 ? 2 : (twob ? 1 : 0);
                    const uint32_t* kl = klist + kd * 2 * kB2Blocks;
                    epi_prep_pass(E, g, gcount, kl, kl + kB2Blocks, klistn[kd], (int)rank, L, C, et, ew, lane,
                                  (dbgon && r == 0) ? dsub + 12 : nullptr);
                }
                const long long c_e1 = clock64();
                const bool okt = wait_t(tfull + slot, use & 1, abort_flag, P.status, w_t);
                if (!bar_and(2, kEpiThreads, okt)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float* pA = php + ((size_t)b * H + cA / dh) * kTileE;
                const float* pB = php + ((size_t)b * H + cB / dh) * kTileE;
                // 1. conversion of this thread's 128 edge columns: o -> fp16 p o, packed in
                // place; the next 16 columns load while these convert
                {
                    const uint32_t ta = tlane + cb, tb2 = tlane + cb + 128;
                    float va[16], wa[16], vb[16], wb[16];
                    tmem_ld16(ta, va);
                    if (two) tmem_ld16(tb2, wa);
#pragma unroll 1
                    for (int j = 0; j < kTileE / 16; j += 2) {
                        tmem_wait_ld();  // columns of chunk j in va / wa
                        tmem_ld16(ta + 16 * (j + 1), vb);
                        if (two) tmem_ld16(tb2 + 16 * (j + 1), wb);
                        epi_convert16(ta, va, pA + 16 * j, j);
                        if (two) epi_convert16(tb2, wa, pB + 16 * j, j);
                        tmem_wait_ld();  // chunk j + 1 in vb / wb
                        if (j + 2 < kTileE / 16) {
                            tmem_ld16(ta + 16 * (j + 2), va);
                            if (two) tmem_ld16(tb2 + 16 * (j + 2), wa);
                        }
                        epi_convert16(ta, vb, pA + 16 * (j + 1), j + 1);
                        if (two) epi_convert16(tb2, wb, pB + 16 * (j + 1), j + 1);
                    }
                }
                tmem_wait_st();
                const long long c_e2 = clock64();
                // 2./3. passes over the node segments
                bool okp = true;
                long long c_dr = 0;
                prepped = false;
                for (int s0 = 0; s0 < nseg; s0 += per) {
                    const int s1 = min(nseg, s0 + per);
                    if (s0 > 0) {  // later passes (many nodes in the tile): list built here
                        const int kd = g.mu > 0 ? 2 : (twob ? 1 : 0);
                        const int q = slot;
                        if (et == 0) epi_reqh(E, q)[0] = epi_build_list(sl_start, kd, s0, s1, epi_req(E, q), epi_reqbp(E, q));
                        asm volatile("bar.sync 2, %0;" ::"n"(kEpiThreads) : "memory");
                        epi_prep_pass(E, g, gcount, epi_req(E, q), epi_reqbp(E, q), epi_reqh(E, q)[0], (int)rank, L, C, et,
                                      ew, lane, (dbgon && r == 0) ? dsub + 12 : nullptr);
                    }
                    tc_fence_before();
                    if (et == 0) *mailbox = slot;
                    asm volatile("bar.sync 2, %0;" ::"n"(kEpiThreads) : "memory");
                    // this CTA's operands of the pass are ready: the even CTA's warp A issues it
                    if (rank == 0) mbar_arrive(a2ready); else mbar_arrive_cluster(at_even(a2ready));
                    const bool okw = okp && wait_t(d2full, d2ph, abort_flag, P.status, w_t);
                    d2ph ^= 1;
                    if (!bar_and(2, kEpiThreads, okw)) { okp = false; break; }
                    tc_fence_after();
                    const long long c_d0 = clock64();
                    // drain: lane c of this warp owns out[node][l3, m'][c]
                    for (int sg = s0; sg < s1; ++sg) {
                        const int node = sl_node[sg];
                        const int nacc = twob ? 2 : 1;
                        for (int a2 = 0; a2 < nacc; ++a2) {
                            const bool vv = a2 == 0 ? vA : vB;
                            if (!vv) continue;  // warp-uniform: this CTA has no rows of that accumulator
                            const int dcol = twob ? d2col((sg - s0) + 2 * a2) : d2col(sg - s0);
                            float v[16];
                            tmem_ld16(tlane + cb + dcol + 16 * rank, v);
                            tmem_wait_ld();
                            const int l3 = a2 == 0 ? l3A : l3B, c = a2 == 0 ? cA : cB;
                            float* o = P.out + ((size_t)node * K + l3 * l3) * C + c;
#pragma unroll
                            for (int mp = 0; mp < 2 * kMaxL + 1; ++mp)
                                if (mp < 2 * l3 + 1) atomicAdd(o + (size_t)mp * C, v[mp]);
                        }
                    }
                    c_dr += clock64() - c_d0;
                    tc_fence_before();
                }
                if (dbgon && r == 0) {
                    const long long c_e3 = clock64();
                    dsub[8] += c_e3 - c_e0;
                    dsub[9] += c_e1 - c_e0;   // first pass prepared (if not during the previous group)
                    dsub[10] += c_e2 - c_e1;  // accumulators awaited and converted
                    dsub[11] += c_e3 - c_e2;  // passes: issue, completion, drains
                }
                if (rank == 0) mbar_arrive(tempty + slot); else mbar_arrive_cluster(at_even(tempty + slot));
                if (!okp) { ok = false; }
                // the next group's first pass (its pairs staged, the other buffer free), while its
                // accumulators are still being computed
                if (ok && gi + 1 < ng) {
                    const bool okd2 = wait_t(dbar + (slot ^ 1), ((gcount + 1) >> 1) & 1, abort_flag, P.status, w_t);
                    if (bar_and(2, kEpiThreads, okd2)) {
                        const TcGroup gn = P.groups[gi + 1];
                        const int pern = (gn.mu == 0 && gn.row0b >= 0) ? 2 : 4;
                        const int kdn = gn.mu > 0 ? 2 : ((gn.mu == 0 && gn.row0b >= 0) ? 1 : 0);
                        const uint32_t* kln = klist + kdn * 2 * kB2Blocks;
                        epi_prep_pass(E, gn, gcount + 1, kln, kln + kB2Blocks, klistn[kdn], (int)rank, L, C, et, ew, lane,
                                      (dbgon && r == 0) ? dsub + 12 : nullptr);
                        (void)pern;
                        prepped = true;
                    } else {
                        ok = false;
                    }
                }
            }
            if (!bar_and(2, kEpiThreads, ok)) { ok = false; break; }
            mbar_arrive(xfree + b);
            mbar_arrive_cluster(at_peer(xfree + b));
        }
        if (P.dbg && r == 0) {
            long long* d = P.dbg + blockIdx.x * kDbgSlots;
            d[8] = w_x; d[9] = w_t; d[10] = clock64() - c_start; d[13] = ntiles; d[22] = dsub[8];
            d[28] = dsub[9]; d[29] = dsub[10]; d[30] = dsub[11]; d[31] = dsub[12];
            d[14] = dsub[13]; d[15] = dsub[14]; d[16] = dsub[15];
        }
#undef E2F_STAGE_GROUP
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
    cluster_sync();  // no MMA of the pair can still touch either CTA's TMEM or shared memory
    if (warp == 12) {
        tc_fence_after();
        tmem_dealloc2(tmem, 512);
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

bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows = 128) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)tc::kKS, box_rows};
    cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(int L, int C, int H, int n_rbf, bool bf16) {
    return bf16 && L >= 1 && L <= kMaxL && C % 128 == 0 && C <= 256 && H <= kMaxHeads && H % 4 == 0 &&
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
        xs = take((size_t)kMaxCtas * 2 * tc::kHalfE * K * C * 2);
        dscr = take((size_t)kMaxCtas * 2 * tc::dglob_pairs() * 4);
        x16 = take((size_t)n_atoms * K * C * 2);
        w16 = take(so2_total(L, C) * 2);
        whT = take((size_t)Gv * kTcMaxRbf * 2);
        gscr = take((size_t)kMaxCtas * 2 * tc::kHalfE * Gv * 2);  // two tile buffers per CTA
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
}  // namespace

void set_tc_kernel_events(void* start, void* stop) {
    g_kernel_ev[0] = static_cast<cudaEvent_t>(start);
    g_kernel_ev[1] = static_cast<cudaEvent_t>(stop);
}

template <int L>
static cudaError_t launch_tc(const tc::TcParams& P, const tc::TcMaps& T, int grid, cudaStream_t s) {
    const size_t smem = tc::SmemLayout(L, P.C, P.H, P.n_rbf).total + 1024;
    cudaError_t e = cudaFuncSetAttribute(tc::k_attn_tc<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // CTA pairs: clusters of two along x, sharing tcgen05.mma.cta_group::2
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)grid);
    lc.blockDim = dim3(tc::kThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&lc, tc::k_attn_tc<L>, P, T);
}

cudaError_t run_attention_tc(const AttnArgs& a, void* tc_ws, cudaStream_t s, const CellLists* cl) {
    const int L = a.L, C = a.C, H = a.H, K = n_sh(L), N = a.n_atoms;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    int cap = kMaxCtas;
    if (const char* env = getenv("E2F_TC_MAX_CTAS")) {  // launch-shape override (tests): fewer, longer CTAs
        const int v = atoi(env);
        if (v > 0 && v < cap) cap = v;
    }
    const int npairs = std::max(1, std::min(sms, cap) / 2);
    const int grid = 2 * npairs;
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
    const size_t qk_smem = (32 * C + tc::kQkRows * (C + 1)) * 4;
    e = cudaFuncSetAttribute(tc::k_qk_tiled, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qk_smem);
    if (e != cudaSuccess) return e;
    count_launch();
    tc::k_qk_tiled<<<(N + 31) / 32, 256, qk_smem, s>>>(static_cast<const __nv_bfloat16*>(a.x), N, K, C, a.Wq, a.Wk,
                                                       a.q, a.k);
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
    tc::k_partition<<<(npairs + 1 + 127) / 128, 128, 0, s>>>(a.row_ptr, N, npairs, part);
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
    if (const char* env = getenv("E2F_TC_TIMERS")) {
        if (atoi(env) > 0) {
            P.dbg = dbg;
            e = cudaMemsetAsync(dbg, 0, kTcDebugBytes, s);
            if (e != cudaSuccess) return e;
        }
    }
    // groups of M = 256 rows (rows r0 .. r0 + 127 in the even CTA, r0 + 128 .. in the odd one):
    // m = 0 feature blocks two at a time; then (o+, o-) per 256 features for m >= 1
    int ng = 0;
    const int n0 = (L + 1) * C;
    for (int r0 = 0; r0 < n0; r0 += 512) {
        tc::TcGroup g{};
        g.mu = 0; g.row0 = r0; g.row0b = (r0 + 256 < n0) ? r0 + 256 : -1; g.klen = n0; g.xoff0 = 0; g.xoff1 = 0;
        g.wa = 0; g.wb = 0;
        P.groups[ng++] = g;
    }
    int koff = n0;
    for (int mu = 1; mu <= a.M; ++mu) {  // |m| > M: no message (truncated layer)
        const int nm = (L + 1 - mu) * C;
        for (int r0 = 0; r0 < nm; r0 += 256) {
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
    if (!make_map(&T.xs, xs, (uint64_t)K * C, (uint64_t)grid * 2 * tc::kHalfE, tc::kHalfE)) return cudaErrorInvalidValue;

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
