// Internal interface between the C-ABI entry points and the attention kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"

namespace e2f {

// Packed SO(2) weight blocks: A(0) of side (L+1)C, then A(m), B(m) of side
// (L+1-m)C for m = 1..L. which = 0 selects A(m), 1 selects B(m).
__host__ __device__ inline size_t so2_offset(int L, int C, int m, int which) {
    size_t n0 = (size_t)(L + 1) * C;
    size_t off = n0 * n0;
    if (m == 0) return 0;
    for (int k = 1; k < m; ++k) {
        size_t n = (size_t)(L + 1 - k) * C;
        off += 2 * n * n;
    }
    size_t n = (size_t)(L + 1 - m) * C;
    return off + (which ? n * n : 0);
}

// values in the packed weights of a layer whose maps stop at |m| = M
__host__ __device__ inline size_t so2_total(int L, int C, int M) {
    return so2_offset(L, C, M + 1, 0);
}
__host__ __device__ inline size_t so2_total(int L, int C) { return so2_total(L, C, L); }

// effective truncation order of a configuration
inline int effective_mmax(int L, int m_max) { return (m_max < 0 || m_max > L) ? L : m_max; }

struct AttnArgs {
    int L, C, H, n_rbf;
    int M;  // SO(2) maps for |m| <= M
    float cutoff;
    bool bf16;
    int n_atoms;
    int64_t n_pairs;
    Box box;
    const float* pos;
    const int32_t* row_ptr;
    const int32_t* col;
    const void* x;
    const float* Wq;
    const float* Wk;
    const float* Wrad;
    const void* Wso2;
    float* out;
    // workspace pieces
    int* status;
    float* q;
    float* k;
    float* Wt;
};

cudaError_t run_attention_simt(const AttnArgs& a, cudaStream_t s);
// q = W_q x[l=0], k = W_k x[l=0]; packed SO(2) weights -> fp32 with each block transposed
cudaError_t qk_project(const void* x, bool bf16, int n_atoms, int K, int C, const float* Wq, const float* Wk,
                       float* q, float* k, cudaStream_t s);
cudaError_t repack_so2_f32(const void* w, bool bf16, int L, int C, int M, float* out, cudaStream_t s);

// Backward pass: the forward's arguments (a.out unused; a.q, a.k, a.Wt are
// workspace) plus dLoss/dout and the gradient outputs (gWq, gWk, gWso2 may be
// null: not computed).
struct BwdArgs {
    AttnArgs fwd;
    const float* grad_out;
    float* lse;
    float* beta;
    float* gq;
    float* gk;
    float* gpos;
    float* gx;
    float* gWq;
    float* gWk;
    float* gWrad;
    float* gWso2;
    float* gWpart;  // bwd_partial_bytes(L, C, M) of scratch for gWso2
    void* w16;      // bf16 storage: 4 so2_total(L, C, M) bytes for fp16 copies of W_so2
    void* ops;      // bf16 storage: bwd_ops_bytes(...) of scratch for the weight-gradient operands
    int* status;    // device status word (cleared by the caller)
};
bool bwd_supported(int L, int C, int H, int n_rbf);
size_t bwd_partial_bytes(int L, int C, int M);
// bf16 storage: the per-chunk operand rows of the SO(2) weight gradient
size_t bwd_ops_bytes(int64_t n_pairs, int L, int C);
cudaError_t run_attention_bwd(const BwdArgs& b, cudaStream_t s);
struct CellLists;
// cl != nullptr: fused traversal (a.row_ptr = per-slot offsets in cell order, a.col unused)
cudaError_t run_attention_tc(const AttnArgs& a, void* tc_ws, cudaStream_t s, const CellLists* cl = nullptr);
void set_tc_kernel_events(void* start, void* stop);
// Debug and test controls of the tensor-core kernel (process-wide): max_ctas > 0
// caps the persistent CTAs, timers != 0 records role cycle counters, drop_arrive
// != 0 makes CTA 0 withhold one producer arrival on its first tile.
void set_tc_debug(int max_ctas, int timers, int drop_arrive);
cudaError_t run_edge_wigner(const float* r, int64_t n, int L, float* out, float* frames, cudaStream_t s);

}  // namespace e2f
