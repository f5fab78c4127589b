// Parameters of the tcgen05 attention path (see attention_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "cell_grid.cuh"
#include "common.cuh"

namespace e2f {

constexpr int kMaxHeads = 16;   // tensor-core path: H <= 16
constexpr int kMaxRbf = 32;
constexpr int kTcMaxRbf = 16;   // tensor-core path: the radial gate is one k=16 mma
constexpr int kMaxCtas = 160;   // persistent CTAs (one per SM; B200 has 148)
constexpr int kDbgSlots = 32;                                         // counters per CTA
constexpr size_t kTcDebugBytes = (size_t)kMaxCtas * kDbgSlots * 8;  // per-CTA role timers

struct StatsParams {
    int n_atoms, C, H, n_rbf, G;
    float cutoff;
    Box box;
    const float* pos;
    const int32_t* row_ptr;
    const int32_t* col;
    const float* q;
    const float* k;
    const float* Wrad;
    float* lse;
};

namespace tc {

constexpr int kMaxGroups = 32;

// One MMA group: up to two 128-row accumulators fed by one K loop.
//   mu >= 1: o+ (TMEM cols 0-127) and o- (128-255) for rows [row0, row0+128)
//            of A(mu)/B(mu) (tensor maps wa/wb); features x+ at xoff0, x- at xoff1
//   mu == 0: rows row0 and row0b (-1: none) of A(0) (map wa); features at xoff0
struct TcGroup {
    int mu, row0, row0b, klen, xoff0, xoff1, wa, wb;
};

struct TcParams {
    int C, H, n_rbf, G;
    int M;      // SO(2) maps for |m| <= M
    int cells;  // fused traversal: row_ptr is per node slot in cell order, neighbours from cv
    CellView cv;
    float cutoff;
    Box box;
    const float* pos;
    const int32_t* row_ptr;
    const int32_t* col;
    const __half* x;       // features in fp16, scaled by scale[0] (an exact power of two)
    const __half* whT;     // value-gate weights, fp16, [(L+1)C][16] (radial index innermost, zero padded)
    __half* gscr;          // per-CTA value-gate scratch [n_ctas][2 tile buffers][128][(L+1)C]
    const float* scale;    // [0] feature scale s, [1] 1/s
    const float* q;
    const float* k;
    const float* lse;
    const float* Wrad;
    const int32_t* part;
    __half* xs;
    __half2* dscr;   // per-CTA Wigner pair blocks (fp16x2), two tile buffers per CTA
    float* out;
    int* status;
    long long* dbg;  // per-CTA role cycle counters, or null
    int drop_arrive; // test hook: CTA 0 withholds one producer arrival on its first tile
    int n_groups;
    TcGroup groups[kMaxGroups];
};

struct TcMaps {
    CUtensorMap w[2 * kMaxL + 1];  // A(0), A(1), B(1), ..., A(L), B(L)
    CUtensorMap xs;                // rotated-feature scratch
};

}  // namespace tc

bool tc_supported(int L, int C, int H, int n_rbf, bool bf16);
size_t tc_workspace_bytes(int64_t n_atoms, int L, int C, int H);

}  // namespace e2f
