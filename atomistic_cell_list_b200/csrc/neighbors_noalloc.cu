// Neighbour build with its scratch in a fixed device array of this library.
//
// Some callers cannot allocate device memory at the moment they need a
// neighbour list: a host program embedded in another runtime whose caching
// allocator already owns nearly all of HBM, or a caller with a latency bound
// that cannot take the device-wide synchronisation of cudaMalloc/cudaFree.
// This entry point serves them: it runs the same kernels as
// e2f_build_neighbors, with the scratch taken from a static __device__
// array instead of a caller workspace, and it allocates nothing itself (no
// cudaMalloc, no allocating library).
#include "common.cuh"

namespace e2f {
namespace {

static_assert(E2F_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte granules");

// Module memory: placed when the module is loaded, one copy per device
// context.
__device__ __align__(256) unsigned char g_nbr_scratch[E2F_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch in the context current on this thread. In
// host code g_nbr_scratch names a host-side stand-in, so the address is
// asked for on every call: a symbol's device address belongs to the context
// the module was loaded in, and a cached one would outlive a device reset
// or a switch to another context on the same device. The lookup is a host
// call; the first one in a context may load the module.
cudaError_t scratch_for_current_context(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_nbr_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace e2f

using namespace e2f;

extern "C" e2f_status e2f_build_neighbors_noalloc(const float* pos, int64_t n_atoms, const float* box_host,
                                                  float cutoff, const int32_t* graph_ptr, int32_t n_graphs,
                                                  int32_t* row_ptr, int32_t* col, int64_t col_capacity,
                                                  int64_t* n_pairs_host, void* stream) {
    if (n_atoms < 0 || !(cutoff > 0.f)) return E2F_ERR_INVALID_ARG;
    // problems whose scratch would not fit are refused before anything runs
    const size_t need = e2f_neighbors_workspace_size(n_atoms, box_host, cutoff, graph_ptr ? n_graphs : 1);
    if (need > (size_t)E2F_NOALLOC_SCRATCH_BYTES) return E2F_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if (scratch_for_current_context(&scratch) != cudaSuccess || !scratch) return E2F_ERR_CUDA;
    // e2f_build_neighbors clears, on `stream`, every scratch word that must
    // start at zero (the flag word, the bucket counts, the degree sentinel)
    // before its first kernel, so what an earlier call left there is harmless.
    return e2f_build_neighbors(pos, n_atoms, box_host, cutoff, graph_ptr, n_graphs, row_ptr, col, col_capacity,
                               n_pairs_host, scratch, (size_t)E2F_NOALLOC_SCRATCH_BYTES, stream);
}
