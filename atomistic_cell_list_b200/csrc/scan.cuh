// Multi-level exclusive prefix sum of uint32 values (used by the cell-list
// counting sort and for row offsets). Each level scans 4096-element tiles
// with one 256-thread block and scans the tile totals one level up.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace e2f {

constexpr int kScanThreads = 256;
constexpr int kScanItems = 16;
constexpr size_t kScanTile = (size_t)kScanThreads * kScanItems;

inline size_t scan_tmp_bytes(size_t n) {
    size_t nb = (n + kScanTile - 1) / kScanTile;
    size_t b = (nb * 4 + 255) / 256 * 256;
    return nb > 1 ? b + scan_tmp_bytes(nb) : b;
}

__global__ void __launch_bounds__(kScanThreads)
k_scan_tile(const uint32_t* in, uint32_t* out, size_t n, uint32_t* tile_sums) {
    __shared__ uint32_t wsum[kScanThreads / 32];
    const size_t base = (size_t)blockIdx.x * kScanTile + (size_t)threadIdx.x * kScanItems;
    uint32_t v[kScanItems];
    uint32_t s = 0;
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        v[k] = (base + k < n) ? in[base + k] : 0u;
        s += v[k];
    }
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
    }
    if (lane == 31) wsum[w] = inc;
    __syncthreads();
    if (w == 0) {
        uint32_t x = lane < kScanThreads / 32 ? wsum[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += t;
        }
        if (lane < kScanThreads / 32) wsum[lane] = x;  // inclusive warp totals
    }
    __syncthreads();
    uint32_t run = inc - s + (w > 0 ? wsum[w - 1] : 0u);
#pragma unroll
    for (int k = 0; k < kScanItems; ++k) {
        if (base + k < n) out[base + k] = run;
        run += v[k];
    }
    if (threadIdx.x == kScanThreads - 1) tile_sums[blockIdx.x] = run;
}

__global__ void k_scan_add(uint32_t* out, size_t n, const uint32_t* tile_off) {
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] += tile_off[i / kScanTile];
}

// in may equal out. tmp must hold scan_tmp_bytes(n) bytes.
inline cudaError_t exclusive_scan_u32(const uint32_t* in, uint32_t* out, size_t n, void* tmp,
                                      cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const size_t nb = (n + kScanTile - 1) / kScanTile;
    uint32_t* sums = static_cast<uint32_t*>(tmp);
    count_launch();
    k_scan_tile<<<(unsigned)nb, kScanThreads, 0, stream>>>(in, out, n, sums);
    if (nb > 1) {
        char* next = static_cast<char*>(tmp) + (nb * 4 + 255) / 256 * 256;
        cudaError_t e = exclusive_scan_u32(sums, sums, nb, next, stream);
        if (e != cudaSuccess) return e;
        count_launch();
        k_scan_add<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(out, n, sums);
    }
    return cudaGetLastError();
}

}  // namespace e2f
