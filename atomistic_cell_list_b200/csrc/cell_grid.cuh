// Cell grid shared by the neighbour build and the fused-traversal attention:
// the exact fp32 pair predicate, the cell of a point, the bucket of a cell
// and the 27-cell stencil (see include/e2f.h, neighbour list).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"

namespace e2f {

constexpr float kCellSlack = 1.0e-3f;

enum : int { kFlagNonFinite = 1, kFlagBadGraph = 2, kFlagStale = 4 };

// Periodic grids use cells at least half the search radius wide and a
// stencil of 5 cells per axis (all cells of an axis with fewer than five);
// open boundaries hash cells at least the search radius wide and search the
// 3 x 3 x 3 cells around a point.
struct Grid {
    Box box;
    int nc[3];           // periodic: cells per axis
    float cell;          // open: cell side
    uint32_t n_buckets;  // periodic: n_graphs * nc^3; open: power of two
    uint32_t mask;       // open: n_buckets - 1
    int noff[3];         // periodic: stencil cells per axis (5, or nc below five)
    float reach;         // search radius the grid was made for
};

__device__ __forceinline__ bool pair_within(float4 a, float4 b, const Grid& g, float rc2) {
    // the exact sequence of IEEE round-to-nearest operations (no FMA)
    float dx = __fsub_rn(b.x, a.x), dy = __fsub_rn(b.y, a.y), dz = __fsub_rn(b.z, a.z);
    if (g.box.periodic) {
        dx = __fsub_rn(dx, __fmul_rn(g.box.len.x, rintf(__fmul_rn(dx, g.box.inv.x))));
        dy = __fsub_rn(dy, __fmul_rn(g.box.len.y, rintf(__fmul_rn(dy, g.box.inv.y))));
        dz = __fsub_rn(dz, __fmul_rn(g.box.len.z, rintf(__fmul_rn(dz, g.box.inv.z))));
    }
    float d2 = __fadd_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)), __fmul_rn(dz, dz));
    return d2 < rc2;
}

__device__ __forceinline__ void cell_of(float x, float y, float z, const Grid& g, long long c[3]) {
    // fp64 so that the cell of a point never moves by more than the slack
    const double p[3] = {x, y, z};
    if (g.box.periodic) {
        const double len[3] = {g.box.len.x, g.box.len.y, g.box.len.z};
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            double w = p[a] - len[a] * floor(p[a] / len[a]);   // wrapped into [0, len]
            long long k = (long long)(w * (double(g.nc[a]) / len[a]));
            c[a] = k < 0 ? 0 : (k >= g.nc[a] ? g.nc[a] - 1 : k);
        }
    } else {
#pragma unroll
        for (int a = 0; a < 3; ++a) c[a] = (long long)floor(p[a] / double(g.cell));
    }
}

__device__ __forceinline__ uint32_t bucket_of(const long long c[3], int gid, const Grid& g) {
    if (g.box.periodic) {
        long long idx = (((long long)gid * g.nc[2] + c[2]) * g.nc[1] + c[1]) * g.nc[0] + c[0];
        return (uint32_t)idx;
    }
    uint64_t h = (uint64_t)c[0] * 0x9E3779B97F4A7C15ull;
    h ^= (uint64_t)c[1] * 0xC2B2AE3D27D4EB4Full + (h >> 29);
    h ^= (uint64_t)c[2] * 0x165667B19E3779F9ull + (h >> 32);
    h ^= (uint64_t)(uint32_t)gid * 0x27D4EB2F165667C5ull + (h >> 31);
    h ^= h >> 33;
    return (uint32_t)h & g.mask;
}

// periodic: cell index c + offset wrapped into [0, nc); c is in [0, nc) and
// c + offset lies in (-nc, 2 nc) (offsets -2 .. 2 on axes of five or more
// cells, 0 .. nc-1 on smaller ones), so one add or subtract of nc suffices
__device__ __forceinline__ long long wrap_cell(long long c, int nc) {
    return c < 0 ? c + nc : (c >= nc ? c - nc : c);
}

// Read-only view of a cell list (periodic grid or, for open boundaries,
// hashed buckets) for kernels that enumerate neighbours: atoms sorted by
// bucket (float4 x, y, z, graph id), their indices, bucket starts
// (n_buckets + 1).
struct CellView {
    Grid g;
    float rc2;
    const float4* spos;
    const int32_t* sidx;
    const uint32_t* start;
    // Verlet-skin reuse: the positions the lists were built from (slot order),
    // else null. The stencil of slot s is then centred on sref[s]'s cell while
    // the pair test uses the current positions in spos.
    const float4* sref = nullptr;
};

// Periodic stencil cell along axis a, entry k (0 <= k < noff[a]): offsets
// -2 .. 2 on an axis of five or more cells, else every cell of the axis once.
__device__ __forceinline__ long long stencil_cell(long long c, const Grid& g, int a, int k) {
    return wrap_cell(c + k - (g.noff[a] == 5 ? 2 : 0), g.nc[a]);
}

// The stencil's candidates: lane l (< 32) holds one range [st, st + len) of
// sorted positions; a warp scan concatenates the ranges in lane order into
// one candidate sequence t = 0 .. ncand-1, and candidate t sits at sorted
// position base(b) + t for the lane b with excl(b) <= t < incl(b), found by a
// binary search over the lanes. Candidates are loaded 4 x 32 at a time before
// any is tested, so the loads overlap. Neighbours found are numbered from
// `total` on; returns the new total (the same on every lane).
template <typename F>
__device__ __forceinline__ int scan_candidates(const CellView& cv, float4 me, int i, int gid, uint32_t st,
                                               uint32_t len, int total, F& f) {
    constexpr unsigned kAll = 0xffffffffu;
    constexpr int kU = 4;
    const int lane = threadIdx.x & 31;
    uint32_t incl = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(kAll, incl, o);
        if (lane >= o) incl += v;
    }
    const uint32_t ncand = __shfl_sync(kAll, incl, 31);
    const uint32_t base = st - (incl - len);  // modulo 2^32: base + t is the sorted position
    for (uint32_t t0 = 0; t0 < ncand; t0 += 32 * kU) {
        float4 o[kU];
        int jj[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const uint32_t t = t0 + 32 * u + lane;
            int b = 0;  // number of lanes with incl <= t
#pragma unroll
            for (int step = 16; step > 0; step >>= 1)
                if (__shfl_sync(kAll, incl, b + step - 1) <= t) b += step;
            const uint32_t sp = __shfl_sync(kAll, base, b) + t;
            o[u] = me;
            jj[u] = -1;
            if (t < ncand) {
                o[u] = cv.spos[sp];
                jj[u] = cv.sidx[sp];
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const bool hit = jj[u] >= 0 && jj[u] != i && __float_as_int(o[u].w) == gid &&
                             pair_within(me, o[u], cv.g, cv.rc2);
            const unsigned m = __ballot_sync(kAll, hit);
            if (hit) f(total + __popc(m & ((1u << lane) - 1u)), jj[u]);
            total += __popc(m);
        }
    }
    return total;
}

// One warp: enumerates the neighbours j of atom i (at me, in graph gid) in
// stencil order, range by range, atoms of a cell in their stored order;
// calls f(k, j) on the lane that holds the k-th neighbour. Returns the count
// (the same on every lane). The predicate is the neighbour build's: j != i,
// same graph (the w field of the stored positions), fp32 distance test.
// Periodic grids: the stencil is gathered as rows along x. The cells of a
// row are consecutive buckets, so lane r holds row r (one (y, z) pair of
// the stencil) as one range; a row that wraps around the box in x takes a
// second pass for its wrapped part. Open boundaries: lane b holds hashed
// bucket b of the 27 (cells that hash to one bucket are visited once).
// slot >= 0: i sits at sorted slot `slot`; with build-time positions (cv.sref)
// the stencil is centred on that slot's build-time cell.
template <typename F>
__device__ __forceinline__ int warp_neighbors(const CellView& cv, float4 me, int i, F&& f, int gid = 0,
                                             int slot = -1) {
    constexpr unsigned kAll = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    const float4 ctr = (cv.sref != nullptr && slot >= 0) ? cv.sref[slot] : me;
    long long c[3];
    cell_of(ctr.x, ctr.y, ctr.z, cv.g, c);
    const Grid& g = cv.g;
    int total = 0;
    if (g.box.periodic) {
        const int nrow = g.noff[1] * g.noff[2], nc0 = g.nc[0];
        const bool all_x = g.noff[0] < 5;
        const long long x0 = c[0] - 2, x1 = c[0] + 2;
        const int npass = (!all_x && (x0 < 0 || x1 >= nc0)) ? 2 : 1;
        // Trim the stencil to the cells the search sphere reaches (fp64, radius
        // padded by 1e-4 relative): a row (y, z offsets) whose y-z distance from
        // the wrapped centre exceeds the radius is skipped, and a row's x range
        // is cut to the cells within the remaining half-width. Axes of fewer
        // than five cells (every cell visited) are not trimmed.
        long long lo_u = x0, hi_u = x1;
        bool empty = lane >= nrow;
        if (!empty) {
            const double len[3] = {g.box.len.x, g.box.len.y, g.box.len.z};
            const double p[3] = {ctr.x, ctr.y, ctr.z};
            double w[3], d2 = 0.0;
#pragma unroll
            for (int a = 0; a < 3; ++a) w[a] = p[a] - len[a] * floor(p[a] / len[a]);
            const int off[3] = {0, lane % g.noff[1], lane / g.noff[1]};
#pragma unroll
            for (int a = 1; a < 3; ++a) {
                if (g.noff[a] == 5) {
                    const double lc = len[a] / g.nc[a];
                    const double lo = (double)(c[a] + off[a] - 2) * lc;
                    const double d = fmax(fmax(lo - w[a], w[a] - (lo + lc)), 0.0);
                    d2 += d * d;
                }
            }
            const double r = (double)g.reach * (1.0 + 1e-4);
            const double rem = r * r - d2;
            if (rem < 0.0) {
                empty = true;
            } else if (!all_x) {
                const double hx = sqrt(rem), lc = len[0] / nc0;
                const long long a = (long long)floor((w[0] - hx) / lc), b = (long long)floor((w[0] + hx) / lc);
                lo_u = a > x0 ? a : x0;
                hi_u = b < x1 ? b : x1;
            }
        }
        for (int p = 0; p < npass; ++p) {
            uint32_t st = 0, len = 0;
            if (!empty) {
                long long lo, hi;
                if (all_x) { lo = 0; hi = nc0 - 1; }
                else if (p == 0) { lo = lo_u < 0 ? 0 : lo_u; hi = hi_u >= nc0 ? nc0 - 1 : hi_u; }
                else if (x0 < 0) { lo = lo_u + nc0; hi = nc0 - 1; }
                else { lo = 0; hi = hi_u - nc0; }
                if (lo <= hi) {
                    const long long cy = stencil_cell(c[1], g, 1, lane % g.noff[1]);
                    const long long cz = stencil_cell(c[2], g, 2, lane / g.noff[1]);
                    const long long row = (((long long)gid * g.nc[2] + cz) * g.nc[1] + cy) * nc0;
                    st = cv.start[row + lo];
                    len = cv.start[row + hi + 1] - st;
                }
            }
            total = scan_candidates(cv, me, i, gid, st, len, total, f);
        }
        return total;
    }
    // open boundaries: the 27 cells around c, x fastest, hashed; of cells that
    // hash to one bucket only the lowest such lane keeps it
    uint32_t bk = 0;
    if (lane < 27) {
        const long long cc[3] = {c[0] + lane % 3 - 1, c[1] + (lane / 3) % 3 - 1, c[2] + lane / 9 - 1};
        bk = bucket_of(cc, gid, g);
    }
    const unsigned same = __match_any_sync(kAll, lane < 27 ? bk : (0x80000000u | (uint32_t)lane));
    uint32_t st = 0, len = 0;
    if (lane < 27 && __ffs(same) - 1 == lane) {
        st = cv.start[bk];
        len = cv.start[bk + 1] - st;
    }
    return scan_candidates(cv, me, i, gid, st, len, total, f);
}

// Cell lists of one system for the fused attention (built by build_cell_lists
// in neighbors.cu): the view, the per-node edge offsets in bucket order
// (rp[N+1]) and an error flag word. With a Verlet skin > 0 the cells are at
// least cutoff + skin wide and the build-time positions are kept (view.sref);
// refresh_cell_lists then reuses the sort for new positions that moved less
// than skin/2 (else kFlagStale), refreshing the positions and the counts.
struct CellLists {
    CellView view;
    const int32_t* rp;
    int* flags;
};
size_t cell_lists_bytes(int64_t n_atoms, const float* box_host, float cutoff, float skin = 0.f);
cudaError_t build_cell_lists(const float* pos, int n_atoms, const float* box_host, float cutoff, void* ws,
                             CellLists* out, cudaStream_t s, float skin = 0.f);
cudaError_t refresh_cell_lists(const float* pos, int n_atoms, const float* box_host, float cutoff, float skin,
                               void* ws, CellLists* out, cudaStream_t s);

inline bool make_grid(const float* box_host, float cutoff, int n_graphs, int64_t n_atoms, Grid& g) {
    g.box.periodic = box_host != nullptr;
    g.reach = cutoff;
    if (g.box.periodic) {
        g.box.len = make_float3(box_host[0], box_host[1], box_host[2]);
        g.box.inv = make_float3(1.0f / box_host[0], 1.0f / box_host[1], 1.0f / box_host[2]);
        long long total = std::max(1, n_graphs);
        for (int a = 0; a < 3; ++a) {  // cells at least half the radius wide
            int nc = (int)std::floor(double(box_host[a]) / (0.5 * double(cutoff) * (1.0 + kCellSlack)));
            g.nc[a] = std::max(1, std::min(nc, 1024));
        }
        // keep the grid at most 2^26 buckets: coarsen the largest axis
        while (total * g.nc[0] * g.nc[1] * g.nc[2] > (1ll << 26)) {
            int a = (g.nc[0] >= g.nc[1] && g.nc[0] >= g.nc[2]) ? 0 : (g.nc[1] >= g.nc[2] ? 1 : 2);
            g.nc[a] = std::max(1, g.nc[a] / 2);
        }
        for (int a = 0; a < 3; ++a) g.noff[a] = std::min(g.nc[a], 5);
        g.n_buckets = (uint32_t)(total * g.nc[0] * g.nc[1] * g.nc[2]);
        g.mask = 0;
        g.cell = 0.f;
    } else {
        g.box.len = g.box.inv = make_float3(0.f, 0.f, 0.f);
        g.cell = cutoff * (1.0f + kCellSlack);
        uint32_t nb = 64;
        while ((int64_t)nb < 2 * n_atoms && nb < (1u << 28)) nb <<= 1;
        g.n_buckets = nb;
        g.mask = nb - 1;
        for (int a = 0; a < 3; ++a) { g.nc[a] = 0; g.noff[a] = 0; }
    }
    return true;
}


}  // namespace e2f
