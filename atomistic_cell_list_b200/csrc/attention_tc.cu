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
// A and B are read by TMA straight from the caller's packed weights (the
// A operand, K-major); h = the tile's rotated, gated neighbour features (the
// B operand, K-major). One A/B weight tile serves two MMAs (the -B product
// uses the instruction's negate bit), so each weight byte is read once per
// 128 edges. A group = up to two accumulators (o+ and o- of the same
// features, or two feature blocks of m = 0) = 256 TMEM columns; two groups
// in flight let the epilogue drain one while the MMA fills the other.
//
// Warp roles (320 threads):
//   0-3  epilogue: tcgen05.ld of the accumulators; per thread one output
//        feature (l3, c) for all 128 edges: p * D^l3(R)^T restricted to the
//        group's |m| rows (the rotate-back, one block at a time), summed
//        over each node's edges in registers, added to out[node] (a CTA owns
//        its nodes, so the read-modify-write is race-free and deterministic)
//   4-7  producer: per edge the frame, Wigner blocks, radial gate, softmax
//        weight p = exp(a - lse) (statistics from a scalar pre-pass: the
//        logits do not depend on the value path, Eq. 6); then the rotated,
//        gated features for all |m| written once per tile to a per-CTA
//        global scratch (bf16, K-major rows) for TMA to stream
//   8    TMA loads of weight and feature tiles into a 3-stage ring
//   9    tcgen05.mma issue (one thread), commits to the ring and TMEM barriers
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
#include "common.cuh"

namespace e2f {
namespace tc {

// ----------------------------------------------------------------------------
// PTX wrappers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, uint32_t tx) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(tx) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(b)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t gtimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// bar.red.and over a named barrier: every participant learns whether all of
// them may continue, so no thread is left waiting at a barrier alone
__device__ __forceinline__ bool bar_and(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait

// Bounded wait. Returns false when the CTA is aborting (this or another wait
// ran out); the first expiry records the status.
__device__ __forceinline__ bool wait(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* status) {
    if (mbar_try(b, parity)) return true;
    const uint64_t t0 = gtimer();
    while (true) {
        if (mbar_try(b, parity)) return true;
        if (*abort_flag) return false;
        if (gtimer() - t0 > kWaitNs) {
            *abort_flag = 1;
            atomicExch(status, (int)E2F_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

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

// kind::f16 instruction descriptor: D fp32, A and B bf16, both K-major,
// M = 128, N = 128, optional negation of A.
__host__ __device__ constexpr uint32_t idesc_bf16(bool neg_a) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((neg_a ? 1u : 0u) << 13) | ((128u >> 3) << 17) |
           ((128u >> 4) << 24);
}

// ----------------------------------------------------------------------------
// pre-passes
// ----------------------------------------------------------------------------
// Logit of edge (i <- j) for head h (Eq. 6 reading): g_a^h <q_i^h, k_j^h>/sqrt(d).
__device__ __forceinline__ float edge_logit(const float* rho, int n_rbf, const float* Wrad, int G, int gcol,
                                            const float* qi, const float* kj, int dh, float inv_sqrt_dh) {
    float ga = 0.f;
    for (int kb = 0; kb < n_rbf; ++kb) ga = fmaf(rho[kb], Wrad[(size_t)kb * G + gcol], ga);
    float dot = 0.f;
    for (int c = 0; c < dh; ++c) dot = fmaf(qi[c], kj[c], dot);
    return ga * dot * inv_sqrt_dh;
}

// Softmax statistics per node and head, lse = m + log(sum exp(a - m)), by an
// online max/sum over the node's edges (one warp per node).
__global__ void __launch_bounds__(256) k_softmax_stats(StatsParams P) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= P.n_atoms) return;
    const int i = warp;
    const int H = P.H, C = P.C, dh = C / H, G = P.G;
    const float inv = rsqrtf((float)dh);
    float m[kMaxHeads], s[kMaxHeads];
#pragma unroll
    for (int h = 0; h < kMaxHeads; ++h) { m[h] = -INFINITY; s[h] = 0.f; }
    const int e0 = P.row_ptr[i], e1 = P.row_ptr[i + 1];
    for (int e = e0 + lane; e < e1; e += 32) {
        const int j = P.col[e];
        float3 r = edge_vec(P.pos, i, j, P.box);
        const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
        float rho[kMaxRbf];
        for (int kb = 0; kb < P.n_rbf; ++kb) rho[kb] = rbf(d, kb, P.cutoff, P.n_rbf);
#pragma unroll
        for (int h = 0; h < kMaxHeads; ++h) {
            if (h < H) {
                float a = edge_logit(rho, P.n_rbf, P.Wrad, G, G - H + h, P.q + (size_t)i * C + h * dh,
                                     P.k + (size_t)j * C + h * dh, dh, inv);
                float mn = fmaxf(m[h], a);
                s[h] = s[h] * expf(m[h] - mn) + expf(a - mn);
                m[h] = mn;
            }
        }
    }
#pragma unroll
    for (int h = 0; h < kMaxHeads; ++h) {
        if (h < H) {
            float mh = m[h], sh = s[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                float mo = __shfl_xor_sync(0xffffffffu, mh, o), so = __shfl_xor_sync(0xffffffffu, sh, o);
                float mn = fmaxf(mh, mo);
                float sa = (mh == -INFINITY) ? 0.f : sh * expf(mh - mn);
                float sb = (mo == -INFINITY) ? 0.f : so * expf(mo - mn);
                mh = mn;
                sh = sa + sb;
            }
            if (lane == 0) P.lse[(size_t)i * H + h] = (e1 > e0) ? mh + logf(sh) : 0.f;
        }
    }
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
// main kernel
// ----------------------------------------------------------------------------
constexpr int kTileE = 128;
constexpr int kKS = 32;                       // K per ring stage
constexpr int kNS = 3;                        // ring stages
constexpr int kSlot = kTileE * kKS * 2;       // 8 KB per operand tile
constexpr int kStage = 4 * kSlot;
constexpr int kThreads = 320;

template <int L>
struct Smem {
    static constexpr int WS = wig_size(L);
    static constexpr int WSP = (WS + 7) & ~7;                 // padded stride (halves)
    static constexpr size_t ring = 0;
    static constexpr size_t dbuf = ring + (size_t)kNS * kStage;
    static constexpr size_t pbuf = dbuf + 2ull * kTileE * WSP * 2;
    static constexpr size_t nid = pbuf + 2ull * kTileE * kMaxHeads * 4;
    static constexpr size_t jn = nid + 2ull * kTileE * 4;
    static constexpr size_t rho = jn + 2ull * kTileE * 4;
    static constexpr size_t bars = rho + (size_t)kTileE * kMaxRbf * 4;
    static constexpr int n_bars = 2 * kNS + 9;
    static constexpr size_t misc = bars + n_bars * 8;
    static constexpr size_t total = misc + 64;
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

template <int L, int L3>
__device__ __forceinline__ void epi_flush(float* out, int node, int c, int C, const float* acc) {
    constexpr int K = n_sh(L);
    float* o = out + ((size_t)node * K + L3 * L3) * C + c;
#pragma unroll
    for (int n = 0; n < 2 * L3 + 1; ++n) o[(size_t)n * C] += acc[n];
}

// One accumulator pair (o+, o-) of block |m| = mu >= 1, or a single
// accumulator (m = 0, pair = false). Thread = output feature (L3, c).
template <int L, int L3>
__device__ __forceinline__ void epi_group(uint32_t tacc, bool pair, int mu, int c, int h, int H, const __half* Db,
                                          const float* pb, const int* nb, float* out, int C) {
    constexpr int WSP = Smem<L>::WSP;
    constexpr int W3 = 2 * L3 + 1;
    float acc[W3];
#pragma unroll
    for (int n = 0; n < W3; ++n) acc[n] = 0.f;
    int cur = -1;
    const int rp = (L3 + mu) * W3, rm = (L3 - mu) * W3;
#pragma unroll 1
    for (int ch = 0; ch < kTileE / 32; ++ch) {
        float vp[32], vm[32];
        tmem_ld32(tacc + ch * 32, vp);
        if (pair) tmem_ld32(tacc + 128 + ch * 32, vm);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            const int e = ch * 32 + q;
            const int node = nb[e];
            if (node != cur) {
                if (cur >= 0) epi_flush<L, L3>(out, cur, c, C, acc);
#pragma unroll
                for (int n = 0; n < W3; ++n) acc[n] = 0.f;
                cur = node;
            }
            if (node < 0) continue;
            const float p = pb[e * kMaxHeads + h];
            const __half* D = Db + (size_t)e * WSP + wig_off(L3);
            const float yp = p * vp[q];
            if (pair) {
                const float ym = p * vm[q];
#pragma unroll
                for (int n = 0; n < W3; ++n)
                    acc[n] = fmaf(__half2float(D[rp + n]), yp, fmaf(__half2float(D[rm + n]), ym, acc[n]));
            } else {
#pragma unroll
                for (int n = 0; n < W3; ++n) acc[n] = fmaf(__half2float(D[rp + n]), yp, acc[n]);
            }
        }
    }
    if (cur >= 0) epi_flush<L, L3>(out, cur, c, C, acc);
    (void)H;
}

template <int L>
__device__ __forceinline__ void epi_dispatch(int l3, uint32_t tacc, bool pair, int mu, int c, int h, int H,
                                             const __half* Db, const float* pb, const int* nb, float* out, int C) {
    switch (l3) {
        case 0: epi_group<L, 0>(tacc, pair, mu, c, h, H, Db, pb, nb, out, C); break;
        case 1: if constexpr (L >= 1) epi_group<L, 1>(tacc, pair, mu, c, h, H, Db, pb, nb, out, C); break;
        case 2: if constexpr (L >= 2) epi_group<L, 2>(tacc, pair, mu, c, h, H, Db, pb, nb, out, C); break;
        case 3: if constexpr (L >= 3) epi_group<L, 3>(tacc, pair, mu, c, h, H, Db, pb, nb, out, C); break;
        case 4: if constexpr (L >= 4) epi_group<L, 4>(tacc, pair, mu, c, h, H, Db, pb, nb, out, C); break;
        default: break;
    }
}

template <int L>
__global__ void __launch_bounds__(kThreads, 1) k_attn_tc(const __grid_constant__ TcParams P,
                                                         const __grid_constant__ TcMaps T) {
    using S = Smem<L>;
    constexpr int K = n_sh(L);
    constexpr int WS = S::WS, WSP = S::WSP;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // operand tiles need 1024-byte alignment in the shared window
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* ring = smem + S::ring;
    __half* dbuf = reinterpret_cast<__half*>(smem + S::dbuf);
    float* pbuf = reinterpret_cast<float*>(smem + S::pbuf);
    int* nid = reinterpret_cast<int*>(smem + S::nid);
    int* jn = reinterpret_cast<int*>(smem + S::jn);
    float* rho = reinterpret_cast<float*>(smem + S::rho);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::bars);
    uint64_t* full = bars;
    uint64_t* empty = bars + kNS;
    uint64_t* tfull = bars + 2 * kNS;
    uint64_t* tempty = tfull + 2;
    uint64_t* xready = tempty + 2;
    uint64_t* xfree = xready + 2;
    uint64_t* fin = xfree + 2;
    uint32_t* tmem_sm = reinterpret_cast<uint32_t*>(smem + S::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = P.C, H = P.H, dh = C / H, G = P.G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kNS; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, 128);
            mbar_init(xready + b, 128);
            mbar_init(xfree + b, 128);
        }
        mbar_init(fin, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 8) {
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
        const int CG = C / 8;
        const size_t KT = (size_t)K * C;
        for (int t = 0; t < ntiles; ++t) {
            const int b = t & 1;
            const bool okw = (t < 2) || wait(xfree + b, ((t - 2) >> 1) & 1, abort_flag, P.status);
            if (!bar_and(1, 128, okw)) break;
            const int e0 = e_begin + t * kTileE;
            const int ne = min(kTileE, e_end - e0);
            __half* Db = dbuf + (size_t)b * kTileE * WSP;
            // P1: one edge per thread
            {
                __half* Dp = Db + (size_t)p * WSP;
                if (p < ne) {
                    const int e = e0 + p;
                    const int j = P.col[e];
                    int lo = n_begin, hi = n_end - 1;  // node i: last n with row_ptr[n] <= e
                    while (lo < hi) {
                        int mid = (lo + hi + 1) >> 1;
                        if (P.row_ptr[mid] <= e) lo = mid; else hi = mid - 1;
                    }
                    const int i = lo;
                    float3 r = edge_vec(P.pos, i, j, P.box);
                    const float d = sqrtf(r.x * r.x + r.y * r.y + r.z * r.z);
                    float R[3][3];
                    edge_frame(r.x / d, r.y / d, r.z / d, R);
                    float D[WS];
                    wigner_blocks<L>(R, D);
#pragma unroll
                    for (int a = 0; a < WS; ++a) Dp[a] = __float2half_rn(D[a]);
                    float rr[kMaxRbf];
                    for (int kb = 0; kb < P.n_rbf; ++kb) {
                        rr[kb] = rbf(d, kb, P.cutoff, P.n_rbf);
                        rho[p * kMaxRbf + kb] = rr[kb];
                    }
                    for (int h = 0; h < H; ++h) {
                        float a = edge_logit(rr, P.n_rbf, P.Wrad, G, G - H + h, P.q + (size_t)i * C + h * dh,
                                             P.k + (size_t)j * C + h * dh, dh, inv_sqrt_dh);
                        pbuf[(b * kTileE + p) * kMaxHeads + h] = expf(a - P.lse[(size_t)i * H + h]);
                    }
                    nid[b * kTileE + p] = i;
                    jn[b * kTileE + p] = j;
                } else {
                    for (int a = 0; a < WS; ++a) Dp[a] = __float2half_rn(0.f);
                    for (int kb = 0; kb < P.n_rbf; ++kb) rho[p * kMaxRbf + kb] = 0.f;
                    for (int h = 0; h < H; ++h) pbuf[(b * kTileE + p) * kMaxHeads + h] = 0.f;
                    nid[b * kTileE + p] = -1;
                    jn[b * kTileE + p] = 0;
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            // P2: rotated, gated features -> scratch row (e), all |m| blocks
            __nv_bfloat16* xrow0 = P.xs + ((size_t)(blockIdx.x * 2 + b) * kTileE) * KT;
            for (int it = p; it < kTileE * CG; it += 128) {
                const int e = it / CG, c0 = (it % CG) * 8;
                __nv_bfloat16* xrow = xrow0 + (size_t)e * KT;
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
                const float* rr = rho + e * kMaxRbf;
                const __half* De = Db + (size_t)e * WSP;
#pragma unroll
                for (int l1 = 0; l1 <= L; ++l1) {
                    float g[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) g[q] = 0.f;
                    for (int kb = 0; kb < P.n_rbf; ++kb) {
                        const float4* wr = reinterpret_cast<const float4*>(P.Wrad + (size_t)kb * G + l1 * C + c0);
                        const float4 w0 = __ldg(wr), w1 = __ldg(wr + 1);
                        const float rk = rr[kb];
                        g[0] = fmaf(rk, w0.x, g[0]); g[1] = fmaf(rk, w0.y, g[1]);
                        g[2] = fmaf(rk, w0.z, g[2]); g[3] = fmaf(rk, w0.w, g[3]);
                        g[4] = fmaf(rk, w1.x, g[4]); g[5] = fmaf(rk, w1.y, g[5]);
                        g[6] = fmaf(rk, w1.z, g[6]); g[7] = fmaf(rk, w1.w, g[7]);
                    }
                    const int w = 2 * l1 + 1;
                    float xv[9][8];
#pragma unroll
                    for (int n = 0; n < 9; ++n) {
                        if (n < w) {
                            const uint4 u = __ldg(reinterpret_cast<const uint4*>(
                                P.x + ((size_t)j * K + l1 * l1 + n) * C + c0));
                            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                float2 f = __bfloat1622float2(h2[q]);
                                xv[n][2 * q] = f.x;
                                xv[n][2 * q + 1] = f.y;
                            }
                        }
                    }
                    const __half* Dl = De + wig_off(l1);
#pragma unroll
                    for (int m = 0; m < 9; ++m) {
                        if (m < w) {
                            float o[8];
#pragma unroll
                            for (int q = 0; q < 8; ++q) o[q] = 0.f;
#pragma unroll
                            for (int n = 0; n < 9; ++n) {
                                if (n < w) {
                                    const float dm = __half2float(Dl[m * w + n]);
#pragma unroll
                                    for (int q = 0; q < 8; ++q) o[q] = fmaf(dm, xv[n][q], o[q]);
                                }
                            }
                            uint4 u;
                            __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                h2[q] = __floats2bfloat162_rn(o[2 * q] * g[2 * q], o[2 * q + 1] * g[2 * q + 1]);
                            *reinterpret_cast<uint4*>(xrow + kpos(l1, m - l1, L, C) + c0) = u;
                        }
                    }
                }
            }
            asm volatile("fence.proxy.async.global;" ::: "memory");
            mbar_arrive(xready + b);
        }
    } else if (warp == 8) {
        // ---------------- TMA ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t ph = 0;
            bool ok = true;
            int pending[kNS];
            for (int s2 = 0; s2 < kNS; ++s2) pending[s2] = -1;
            for (int t = 0; t < ntiles && ok; ++t) {
                const int b = t & 1;
                if (!wait(xready + b, (t >> 1) & 1, abort_flag, P.status)) { ok = false; break; }
                const int rowT = (blockIdx.x * 2 + b) * kTileE;
                for (int gi = 0; gi < ng && ok; ++gi) {
                    const TcGroup g = P.groups[gi];
                    for (int kk = 0; kk < g.klen; kk += kKS) {
                        if (!wait(empty + stage, ph ^ 1, abort_flag, P.status)) { ok = false; break; }
                        uint8_t* st = ring + (size_t)stage * kStage;
                        const int ntile = g.mu > 0 ? 4 : (g.row0b >= 0 ? 3 : 2);
                        mbar_arrive_tx(full + stage, ntile * kSlot);
                        if (g.mu > 0) {
                            tma_load_2d(st, &T.w[g.wa], kk, g.row0, full + stage);
                            tma_load_2d(st + kSlot, &T.w[g.wb], kk, g.row0, full + stage);
                            tma_load_2d(st + 2 * kSlot, &T.xs, g.xoff0 + kk, rowT, full + stage);
                            tma_load_2d(st + 3 * kSlot, &T.xs, g.xoff1 + kk, rowT, full + stage);
                        } else {
                            tma_load_2d(st, &T.w[g.wa], kk, g.row0, full + stage);
                            if (g.row0b >= 0) tma_load_2d(st + kSlot, &T.w[g.wa], kk, g.row0b, full + stage);
                            tma_load_2d(st + 2 * kSlot, &T.xs, g.xoff0 + kk, rowT, full + stage);
                        }
                        pending[stage] = (int)ph;
                        if (++stage == kNS) { stage = 0; ph ^= 1; }
                    }
                }
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
    } else if (warp == 9) {
        // ---------------- MMA ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t ph = 0;
            long long gcount = 0;
            bool ok = true;
            constexpr uint32_t ID = idesc_bf16(false), IDN = idesc_bf16(true);
            for (int t = 0; t < ntiles && ok; ++t) {
                for (int gi = 0; gi < ng && ok; ++gi, ++gcount) {
                    const TcGroup g = P.groups[gi];
                    const int slot = (int)(gcount & 1);
                    const uint32_t use = (uint32_t)(gcount >> 1);
                    if (!wait(tempty + slot, (use & 1) ^ 1, abort_flag, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d0 = tmem + slot * 256, d1 = d0 + 128;
                    for (int kk = 0; kk < g.klen; kk += kKS) {
                        if (!wait(full + stage, ph, abort_flag, P.status)) { ok = false; break; }
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
            // every issued MMA completes (bounded wait) before TMEM is released
            umma_commit(fin);
            const uint64_t t0 = gtimer();
            while (!mbar_try(fin, 0) && gtimer() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 0-3, thread = TMEM lane) ----------------
        const int r = threadIdx.x;
        long long gcount = 0;
        bool ok = true;
        for (int t = 0; t < ntiles && ok; ++t) {
            const int b = t & 1;
            if (!wait(xready + b, (t >> 1) & 1, abort_flag, P.status)) { ok = false; break; }
            const __half* Db = dbuf + (size_t)b * kTileE * WSP;
            const float* pb = pbuf + (size_t)b * kTileE * kMaxHeads;
            const int* nb = nid + b * kTileE;
            for (int gi = 0; gi < ng; ++gi, ++gcount) {
                const TcGroup g = P.groups[gi];
                const int slot = (int)(gcount & 1);
                const uint32_t use = (uint32_t)(gcount >> 1);
                if (!wait(tfull + slot, use & 1, abort_flag, P.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tacc = tmem + ((uint32_t)(warp * 32) << 16) + slot * 256;
                if (g.mu > 0) {
                    const int row = g.row0 + r;
                    const int l3 = g.mu + row / C, c = row % C;
                    epi_dispatch<L>(l3, tacc, true, g.mu, c, c / dh, H, Db, pb, nb, P.out, C);
                } else {
                    const int ra = g.row0 + r;
                    epi_dispatch<L>(ra / C, tacc, false, 0, ra % C, (ra % C) / dh, H, Db, pb, nb, P.out, C);
                    if (g.row0b >= 0) {
                        const int rb = g.row0b + r;
                        epi_dispatch<L>(rb / C, tacc + 128, false, 0, rb % C, (rb % C) / dh, H, Db, pb, nb, P.out,
                                        C);
                    }
                }
                tc_fence_before();
                mbar_arrive(tempty + slot);
            }
            if (ok) mbar_arrive(xfree + b);
        }
    }

    // MMA completion before TMEM release: the epilogue consumed every group it
    // waited for; on a normal exit all MMAs are complete. On abort, wait
    // (bounded) for the last commits to land.
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
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
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_supported(int L, int C, int H, int n_rbf, bool bf16) {
    return bf16 && L >= 1 && L <= kMaxL && C % 128 == 0 && C <= 256 && H <= kMaxHeads && H % 4 == 0 &&
           n_rbf <= kMaxRbf;
}

size_t tc_workspace_bytes(int64_t n_atoms, int L, int C, int H) {
    size_t b = 0;
    b += align_up(4 * (size_t)n_atoms * H, 256);                                       // lse
    b += align_up(4 * (size_t)(kMaxCtas + 1), 256);                                    // partition
    b += align_up((size_t)kMaxCtas * 2 * tc::kTileE * n_sh(L) * C * 2, 256);           // feature scratch
    return b;
}

template <int L>
static cudaError_t launch_tc(const tc::TcParams& P, const tc::TcMaps& T, int grid, cudaStream_t s) {
    const size_t smem = tc::Smem<L>::total + 1024;
    cudaError_t e = cudaFuncSetAttribute(tc::k_attn_tc<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    tc::k_attn_tc<L><<<grid, tc::kThreads, smem, s>>>(P, T);
    return cudaGetLastError();
}

cudaError_t run_attention_tc(const AttnArgs& a, void* tc_ws, cudaStream_t s) {
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
    const int grid = std::max(1, std::min(sms, cap));
    char* w = static_cast<char*>(tc_ws);
    float* lse = reinterpret_cast<float*>(w);
    w += align_up(4 * (size_t)N * H, 256);
    int32_t* part = reinterpret_cast<int32_t*>(w);
    w += align_up(4 * (size_t)(kMaxCtas + 1), 256);
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(w);

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
    tc::k_softmax_stats<<<(N + 7) / 8, 256, 0, s>>>(sp);
    count_launch();
    tc::k_partition<<<(grid + 1 + 127) / 128, 128, 0, s>>>(a.row_ptr, N, grid, part);
    e = cudaMemsetAsync(a.out, 0, (size_t)N * K * C * 4, s);
    if (e != cudaSuccess) return e;

    tc::TcParams P{};
    P.C = C; P.H = H; P.n_rbf = a.n_rbf; P.G = (L + 1) * C + H; P.cutoff = a.cutoff; P.box = a.box;
    P.pos = a.pos; P.row_ptr = a.row_ptr; P.col = a.col; P.x = static_cast<const __nv_bfloat16*>(a.x);
    P.q = a.q; P.k = a.k; P.lse = lse; P.Wrad = a.Wrad; P.part = part; P.xs = xs; P.out = a.out;
    P.status = a.status;
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
    for (int mu = 1; mu <= L; ++mu) {
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
    const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.Wso2);
    if (!make_map(&T.w[0], W + so2_offset(L, C, 0, 0), n0, n0)) return cudaErrorInvalidValue;
    for (int mu = 1; mu <= L; ++mu) {
        const int nm = (L + 1 - mu) * C;
        if (!make_map(&T.w[2 * mu - 1], W + so2_offset(L, C, mu, 0), nm, nm)) return cudaErrorInvalidValue;
        if (!make_map(&T.w[2 * mu], W + so2_offset(L, C, mu, 1), nm, nm)) return cudaErrorInvalidValue;
    }
    if (!make_map(&T.xs, xs, (uint64_t)K * C, (uint64_t)grid * 2 * tc::kTileE)) return cudaErrorInvalidValue;

    switch (L) {
        case 1: return launch_tc<1>(P, T, grid, s);
        case 2: return launch_tc<2>(P, T, grid, s);
        case 3: return launch_tc<3>(P, T, grid, s);
        case 4: return launch_tc<4>(P, T, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace e2f
