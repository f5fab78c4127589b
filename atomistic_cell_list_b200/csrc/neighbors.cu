// Cell-list neighbour build for libe2f (see include/e2f.h).
//
// Pipeline (one stream, one host synchronisation to read E):
//   1 prep      per atom: finite check, graph id, cell -> bucket, rank in
//               bucket (atomic count)
//   2 scan      bucket counts -> bucket starts
//   3 scatter   atoms sorted by bucket: float4 (x, y, z, graph id), index
//   4 count     one warp per atom scans its 27 neighbouring buckets with
//               the exact fp32 predicate -> degree
//   5 scan      degrees -> row_ptr; E and error flags copied to the host
//   6 fill      same scan, neighbours gathered in shared memory, bitonic
//               sorted, written ascending
// Periodic boxes use a direct grid of n_c^3 cells per graph (cells at least
// cutoff*(1+1e-3) wide); open boundaries hash (graph, cell) into 2^k
// buckets and drop repeated buckets from the 27-cell stencil, so a
// collision only adds candidates that the predicate then rejects.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>

#include "cell_grid.cuh"
#include "common.cuh"
#include "scan.cuh"

namespace e2f {
namespace {

constexpr int kSortCap = 1024;   // rows up to this many neighbours sort in shared memory
constexpr int kWarpsPerBlock = 4;
__device__ __forceinline__ int graph_id(const int32_t* gp, int n_graphs, int i) {
    if (!gp) return 0;
    int lo = 0, hi = n_graphs - 1;  // last g with gp[g] <= i
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(gp + mid) <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void k_check_graphs(const int32_t* gp, int n_graphs, int n_atoms, int* flags) {
    int g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g > n_graphs) return;
    int v = gp[g];
    bool bad = (g == 0 && v != 0) || (g == n_graphs && v != n_atoms) || v < 0 || v > n_atoms ||
               (g < n_graphs && gp[g + 1] < v);
    if (bad) atomicOr(flags, kFlagBadGraph);
}

__global__ void k_prep(const float* __restrict__ pos, int n, const int32_t* gp, int n_graphs, Grid g,
                       uint32_t* key, uint32_t* rank, uint32_t* count, int* flags) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float x = pos[3 * i], y = pos[3 * i + 1], z = pos[3 * i + 2];
    uint32_t b = 0;
    if (!(isfinite(x) && isfinite(y) && isfinite(z))) {
        atomicOr(flags, kFlagNonFinite);
    } else {
        long long c[3];
        cell_of(x, y, z, g, c);
        b = bucket_of(c, graph_id(gp, n_graphs, i), g);
    }
    key[i] = b;
    rank[i] = atomicAdd(count + b, 1u);
}

__global__ void k_scatter(const float* __restrict__ pos, int n, const int32_t* gp, int n_graphs,
                          const uint32_t* key, const uint32_t* rank, const uint32_t* start,
                          float4* sorted_pos, int32_t* sorted_idx) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    uint32_t s = start[key[i]] + rank[i];
    sorted_pos[s] = make_float4(pos[3 * i], pos[3 * i + 1], pos[3 * i + 2],
                                __int_as_float(graph_id(gp, n_graphs, i)));
    sorted_idx[s] = i;
}

// One warp per atom. MODE 0: count neighbours into deg[i]. MODE 1: write the
// row ascending at col[row_ptr[i] ...].
template <int MODE>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
k_pairs(const float* __restrict__ pos, int n, int nq, const int32_t* gp, int n_graphs, Grid g, float rc2,
        const uint32_t* __restrict__ start, const float4* __restrict__ sorted_pos,
        const int32_t* __restrict__ sorted_idx, int32_t* deg, const int32_t* __restrict__ row_ptr,
        int32_t* col) {
    __shared__ int32_t buf[kWarpsPerBlock][kSortCap];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int i = blockIdx.x * kWarpsPerBlock + wib;
    if (i >= n) return;
    if (i >= nq) {  // not a query row: an empty row (its atom is still a candidate neighbour)
        if (MODE == 0 && lane == 0) deg[i] = 0;
        return;
    }
    const int gid = graph_id(gp, n_graphs, i);
    const float4 me = make_float4(pos[3 * i], pos[3 * i + 1], pos[3 * i + 2], __int_as_float(gid));
    int row0 = 0, rlen = 0;
    if (MODE == 1) { row0 = row_ptr[i]; rlen = row_ptr[i + 1] - row0; }
    const bool in_smem = (MODE == 1) && rlen <= kSortCap;
    const CellView cv{g, rc2, sorted_pos, sorted_idx, start};
    const int total = warp_neighbors(
        cv, me, i,
        [&](int slot, int j) {
            if (MODE == 1 && slot < rlen) {  // equal counts in both passes; guard anyway
                if (in_smem) buf[wib][slot] = j; else col[row0 + slot] = j;
            }
        },
        gid);
    if (MODE == 0) {
        if (lane == 0) deg[i] = total;
        return;
    }
    __syncwarp();
    if (in_smem) {
        int P = 1;
        while (P < rlen) P <<= 1;
        for (int t = rlen + lane; t < P; t += 32) buf[wib][t] = 0x7fffffff;
        __syncwarp();
        for (int k = 2; k <= P; k <<= 1)
            for (int jj = k >> 1; jj > 0; jj >>= 1) {
                for (int t = lane; t < P; t += 32) {
                    int u = t ^ jj;
                    if (u > t) {
                        int a = buf[wib][t], bb = buf[wib][u];
                        bool up = (t & k) == 0;
                        if ((a > bb) == up) { buf[wib][t] = bb; buf[wib][u] = a; }
                    }
                }
                __syncwarp();
            }
        for (int t = lane; t < rlen; t += 32) col[row0 + t] = buf[wib][t];
        return;
    }
    // very dense row: odd-even transposition sort in place (global memory)
    int32_t* r = col + row0;
    for (int phase = 0; phase < rlen; ++phase) {
        for (int t = 2 * lane + (phase & 1); t + 1 < rlen; t += 64) {
            int a = r[t], bb = r[t + 1];
            if (a > bb) { r[t] = bb; r[t + 1] = a; }
        }
        __syncwarp();
        __threadfence_block();
    }
}

struct NbrWs {
    int* flags;
    uint32_t* key;
    uint32_t* rank;
    uint32_t* count;     // n_buckets + 1
    float4* sorted_pos;
    int32_t* sorted_idx;
    int32_t* deg;        // n + 1
    void* scan_tmp;
    size_t bytes;
};

NbrWs carve(void* base, int64_t n, uint32_t n_buckets) {
    NbrWs w{};
    size_t o = 0;
    auto take = [&](size_t b) { size_t r = o; o = align_up(o + b, 256); return r; };
    char* p = static_cast<char*>(base);
    size_t o_flags = take(256);
    size_t o_key = take(4 * (size_t)n), o_rank = take(4 * (size_t)n);
    size_t o_count = take(4 * ((size_t)n_buckets + 1));
    size_t o_spos = take(16 * (size_t)n), o_sidx = take(4 * (size_t)n);
    size_t o_deg = take(4 * ((size_t)n + 1));
    size_t tmp = std::max(scan_tmp_bytes((size_t)n_buckets + 1), scan_tmp_bytes((size_t)n + 1));
    size_t o_tmp = take(tmp);
    w.bytes = o;
    if (p) {
        w.flags = (int*)(p + o_flags);
        w.key = (uint32_t*)(p + o_key);
        w.rank = (uint32_t*)(p + o_rank);
        w.count = (uint32_t*)(p + o_count);
        w.sorted_pos = (float4*)(p + o_spos);
        w.sorted_idx = (int32_t*)(p + o_sidx);
        w.deg = (int32_t*)(p + o_deg);
        w.scan_tmp = p + o_tmp;
    }
    return w;
}

}  // namespace
}  // namespace e2f

namespace e2f {
namespace {

// Atoms of each bucket in index order (the scatter's order comes from atomic
// ranks): insertion sort, one thread per bucket (buckets hold ~10 atoms).
__global__ void k_sort_buckets(const uint32_t* __restrict__ start, uint32_t n_buckets, float4* spos,
                               int32_t* sidx) {
    const uint32_t b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= n_buckets) return;
    const uint32_t s0 = start[b], s1 = start[b + 1];
    for (uint32_t s = s0 + 1; s < s1; ++s) {
        const int32_t key = sidx[s];
        const float4 v = spos[s];
        uint32_t t = s;
        while (t > s0 && sidx[t - 1] > key) {
            sidx[t] = sidx[t - 1];
            spos[t] = spos[t - 1];
            --t;
        }
        sidx[t] = key;
        spos[t] = v;
    }
}

// Degree of each atom, in bucket order: one warp per sorted position.
__global__ void __launch_bounds__(128) k_count_sorted(CellView cv, int n, int32_t* deg) {
    const int s = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (s >= n) return;
    const int cnt = warp_neighbors(cv, cv.spos[s], cv.sidx[s], [](int, int) {}, 0, s);
    if ((threadIdx.x & 31) == 0) deg[s] = cnt;
}

}  // namespace

// Verlet-skin refresh of one slot: the current position of atom sidx[s]
// replaces the stored one; a displacement from the build-time position
// (minimum image) above skin/2, or a non-finite position, is flagged.
__global__ void k_refresh(const float* __restrict__ pos, int n, Grid g, float half_skin2,
                          const int32_t* __restrict__ sidx, const float4* __restrict__ sref, float4* spos,
                          int* flags) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= n) return;
    const int i = sidx[s];
    const float x = pos[3 * i], y = pos[3 * i + 1], z = pos[3 * i + 2];
    const float4 r = sref[s];
    if (!(isfinite(x) && isfinite(y) && isfinite(z))) atomicOr(flags, kFlagNonFinite);
    float dx = x - r.x, dy = y - r.y, dz = z - r.z;
    if (g.box.periodic) {
        dx -= g.box.len.x * rintf(dx * g.box.inv.x);
        dy -= g.box.len.y * rintf(dy * g.box.inv.y);
        dz -= g.box.len.z * rintf(dz * g.box.inv.z);
    }
    if (!(dx * dx + dy * dy + dz * dz <= half_skin2)) atomicOr(flags, kFlagStale);
    spos[s] = make_float4(x, y, z, r.w);
}

// Workspace of the cell lists: the neighbour build's arrays, rp[N+1] and,
// with a skin, the build-time positions in slot order.
static size_t rp_offset(int64_t n, const Grid& g) { return carve(nullptr, n, g.n_buckets).bytes; }
static size_t sref_offset(int64_t n, const Grid& g) { return rp_offset(n, g) + align_up(4 * ((size_t)n + 1), 256); }

size_t cell_lists_bytes(int64_t n_atoms, const float* box_host, float cutoff, float skin) {
    Grid g;
    make_grid(box_host, cutoff + skin, 1, n_atoms, g);
    return sref_offset(n_atoms, g) + (skin > 0.f ? align_up(16 * (size_t)n_atoms, 256) : 0);
}

// degrees in bucket order, then rp = their exclusive scan
static cudaError_t count_and_scan(const CellView& cv, int n, const NbrWs& w, int32_t* rp, cudaStream_t s) {
    count_launch();
    k_count_sorted<<<(n + 3) / 4, 128, 0, s>>>(cv, n, w.deg);
    cudaError_t e = cudaMemsetAsync(w.deg + n, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    return exclusive_scan_u32(reinterpret_cast<uint32_t*>(w.deg), reinterpret_cast<uint32_t*>(rp), (size_t)n + 1,
                              w.scan_tmp, s);
}

cudaError_t build_cell_lists(const float* pos, int n, const float* box_host, float cutoff, void* ws,
                             CellLists* out, cudaStream_t s, float skin) {
    Grid g;
    make_grid(box_host, cutoff + skin, 1, n, g);
    NbrWs w = carve(ws, n, g.n_buckets);
    int32_t* rp = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + rp_offset(n, g));
    float4* sref = skin > 0.f ? reinterpret_cast<float4*>(static_cast<char*>(ws) + sref_offset(n, g)) : nullptr;
    cudaError_t e = cudaMemsetAsync(w.flags, 0, 256, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(w.count, 0, 4 * ((size_t)g.n_buckets + 1), s);
    if (e != cudaSuccess) return e;
    const int tb = 256, nbk = (n + tb - 1) / tb;
    count_launch();
    k_prep<<<nbk, tb, 0, s>>>(pos, n, nullptr, 1, g, w.key, w.rank, w.count, w.flags);
    e = exclusive_scan_u32(w.count, w.count, (size_t)g.n_buckets + 1, w.scan_tmp, s);
    if (e != cudaSuccess) return e;
    count_launch();
    k_scatter<<<nbk, tb, 0, s>>>(pos, n, nullptr, 1, w.key, w.rank, w.count, w.sorted_pos, w.sorted_idx);
    count_launch();
    k_sort_buckets<<<(g.n_buckets + 255) / 256, 256, 0, s>>>(w.count, g.n_buckets, w.sorted_pos, w.sorted_idx);
    if (sref) {
        e = cudaMemcpyAsync(sref, w.sorted_pos, 16 * (size_t)n, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return e;
    }
    CellView cv{g, cutoff * cutoff, w.sorted_pos, w.sorted_idx, w.count, sref};
    e = count_and_scan(cv, n, w, rp, s);
    if (e != cudaSuccess) return e;
    out->view = cv;
    out->rp = rp;
    out->flags = w.flags;
    return cudaGetLastError();
}

cudaError_t refresh_cell_lists(const float* pos, int n, const float* box_host, float cutoff, float skin,
                               void* ws, CellLists* out, cudaStream_t s) {
    if (!(skin > 0.f)) return cudaErrorInvalidValue;
    Grid g;
    make_grid(box_host, cutoff + skin, 1, n, g);
    NbrWs w = carve(ws, n, g.n_buckets);
    int32_t* rp = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + rp_offset(n, g));
    float4* sref = reinterpret_cast<float4*>(static_cast<char*>(ws) + sref_offset(n, g));
    cudaError_t e = cudaMemsetAsync(w.flags, 0, 256, s);
    if (e != cudaSuccess) return e;
    count_launch();
    k_refresh<<<(n + 255) / 256, 256, 0, s>>>(pos, n, g, 0.25f * skin * skin, w.sorted_idx, sref, w.sorted_pos,
                                              w.flags);
    CellView cv{g, cutoff * cutoff, w.sorted_pos, w.sorted_idx, w.count, sref};
    e = count_and_scan(cv, n, w, rp, s);
    if (e != cudaSuccess) return e;
    out->view = cv;
    out->rp = rp;
    out->flags = w.flags;
    return cudaGetLastError();
}

}  // namespace e2f

using namespace e2f;

extern "C" size_t e2f_neighbors_workspace_size(int64_t n_atoms, const float* box_host, float cutoff,
                                               int32_t n_graphs) {
    if (n_atoms < 0 || !(cutoff > 0.f)) return 0;
    Grid g;
    make_grid(box_host, cutoff, std::max(1, (int)n_graphs), n_atoms, g);
    return carve(nullptr, n_atoms, g.n_buckets).bytes;
}

namespace e2f {
namespace {
e2f_status build_neighbors(const float* pos, int64_t n_atoms, int64_t n_rows, const float* box_host, float cutoff,
                           const int32_t* graph_ptr, int32_t n_graphs, int32_t* row_ptr, int32_t* col,
                           int64_t col_capacity, int64_t* n_pairs_host, void* workspace, size_t ws_bytes,
                           void* stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (!n_pairs_host || !row_ptr || n_atoms < 0 || n_atoms > INT32_MAX - 1 || !(cutoff > 0.f) ||
        !std::isfinite(cutoff) || col_capacity < 0 || n_rows < 0 || n_rows > n_atoms)
        return E2F_ERR_INVALID_ARG;
    if (n_atoms > 0 && (!pos || !workspace)) return E2F_ERR_INVALID_ARG;
    if (graph_ptr && n_graphs < 1) return E2F_ERR_INVALID_ARG;
    if (col_capacity > 0 && !col) return E2F_ERR_INVALID_ARG;
    if (box_host) {
        for (int a = 0; a < 3; ++a)
            if (!(box_host[a] > 0.f) || !std::isfinite(box_host[a]) || cutoff > 0.5f * box_host[a])
                return E2F_ERR_INVALID_ARG;
    }
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return E2F_ERR_ALIGNMENT;
    const int ng = graph_ptr ? n_graphs : 1;
    const int n = (int)n_atoms;
    if (n == 0) {
        E2F_CUDA_TRY(cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), stream));
        E2F_CUDA_TRY(cudaStreamSynchronize(stream));
        *n_pairs_host = 0;
        return E2F_OK;
    }
    Grid g;
    make_grid(box_host, cutoff, ng, n_atoms, g);
    NbrWs w = carve(workspace, n_atoms, g.n_buckets);
    if (ws_bytes < w.bytes) return E2F_ERR_INVALID_ARG;
    const float rc2 = cutoff * cutoff;  // fp32 product, as in the predicate

    E2F_CUDA_TRY(cudaMemsetAsync(w.flags, 0, 256, stream));
    E2F_CUDA_TRY(cudaMemsetAsync(w.count, 0, 4 * ((size_t)g.n_buckets + 1), stream));
    if (graph_ptr) {
        count_launch();
        k_check_graphs<<<(ng + 1 + 255) / 256, 256, 0, stream>>>(graph_ptr, ng, n, w.flags);
    }
    const int tb = 256, nbk = (n + tb - 1) / tb;
    count_launch();
    k_prep<<<nbk, tb, 0, stream>>>(pos, n, graph_ptr, ng, g, w.key, w.rank, w.count, w.flags);
    E2F_CUDA_TRY(exclusive_scan_u32(w.count, w.count, (size_t)g.n_buckets + 1, w.scan_tmp, stream));
    count_launch();
    k_scatter<<<nbk, tb, 0, stream>>>(pos, n, graph_ptr, ng, w.key, w.rank, w.count, w.sorted_pos,
                                       w.sorted_idx);
    const int wb = (n + kWarpsPerBlock - 1) / kWarpsPerBlock;
    count_launch();
    k_pairs<0><<<wb, 32 * kWarpsPerBlock, 0, stream>>>(pos, n, (int)n_rows, graph_ptr, ng, g, rc2, w.count,
                                                       w.sorted_pos, w.sorted_idx, w.deg, nullptr, nullptr);
    E2F_CUDA_TRY(cudaMemsetAsync(w.deg + n, 0, sizeof(int32_t), stream));
    E2F_CUDA_TRY(exclusive_scan_u32(reinterpret_cast<uint32_t*>(w.deg), reinterpret_cast<uint32_t*>(row_ptr),
                                    (size_t)n + 1, w.scan_tmp, stream));
    int host[2] = {0, 0};
    E2F_CUDA_TRY(cudaMemcpyAsync(&host[0], row_ptr + n, sizeof(int32_t), cudaMemcpyDeviceToHost, stream));
    E2F_CUDA_TRY(cudaMemcpyAsync(&host[1], w.flags, sizeof(int32_t), cudaMemcpyDeviceToHost, stream));
    E2F_CUDA_TRY(cudaStreamSynchronize(stream));
    E2F_CUDA_TRY(cudaGetLastError());
    if (host[1] & kFlagBadGraph) return E2F_ERR_INVALID_ARG;
    if (host[1] & kFlagNonFinite) return E2F_ERR_NONFINITE;
    const int64_t E = (uint32_t)host[0];
    *n_pairs_host = E;
    if (E > col_capacity) return E2F_ERR_CAPACITY;
    if (E > 0) {
        count_launch();
        k_pairs<1><<<wb, 32 * kWarpsPerBlock, 0, stream>>>(pos, n, (int)n_rows, graph_ptr, ng, g, rc2, w.count,
                                                           w.sorted_pos, w.sorted_idx, nullptr, row_ptr, col);
        E2F_CUDA_TRY(cudaGetLastError());
    }
    return E2F_OK;
}
}  // namespace
}  // namespace e2f

extern "C" e2f_status e2f_build_neighbors(const float* pos, int64_t n_atoms, const float* box_host,
                                          float cutoff, const int32_t* graph_ptr, int32_t n_graphs,
                                          int32_t* row_ptr, int32_t* col, int64_t col_capacity,
                                          int64_t* n_pairs_host, void* workspace, size_t ws_bytes,
                                          void* stream) {
    return e2f::build_neighbors(pos, n_atoms, n_atoms, box_host, cutoff, graph_ptr, n_graphs, row_ptr, col,
                                col_capacity, n_pairs_host, workspace, ws_bytes, stream);
}

extern "C" e2f_status e2f_build_neighbors_rows(const float* pos, int64_t n_atoms, int64_t n_rows,
                                               const float* box_host, float cutoff, const int32_t* graph_ptr,
                                               int32_t n_graphs, int32_t* row_ptr, int32_t* col,
                                               int64_t col_capacity, int64_t* n_pairs_host, void* workspace,
                                               size_t ws_bytes, void* stream) {
    return e2f::build_neighbors(pos, n_atoms, n_rows, box_host, cutoff, graph_ptr, n_graphs, row_ptr, col,
                                col_capacity, n_pairs_host, workspace, ws_bytes, stream);
}
