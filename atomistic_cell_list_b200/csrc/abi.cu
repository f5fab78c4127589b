// C-ABI entry points of libe2f.so for the attention path (argument checks,
// workspace layout, dispatch). The neighbour build lives in neighbors.cu.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <unordered_map>

#include "attention.cuh"
#include "cell_grid.cuh"
#include "attention_tc.cuh"
#include "common.cuh"

namespace e2f {
static std::atomic<long long> g_launches{0};
void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace e2f

using namespace e2f;

namespace {

struct AttnWs {
    size_t o_status, o_q, o_k, o_wt, o_tc, bytes;
    bool tc;
};

AttnWs attn_layout(int64_t n_atoms, const e2f_attn_cfg& c) {
    AttnWs w{};
    size_t o = 0;
    auto take = [&](size_t b) { size_t r = o; o = align_up(o + b, 256); return r; };
    w.o_status = take(256);
    w.o_q = take(4 * (size_t)n_atoms * c.C);
    w.o_k = take(4 * (size_t)n_atoms * c.C);
    w.tc = tc_supported(c.L, c.C, c.H, c.n_rbf, c.feat_dtype == E2F_BF16);
    w.o_wt = w.tc ? 0 : take(4 * so2_total(c.L, c.C, effective_mmax(c.L, c.m_max)));
    w.o_tc = w.tc ? take(tc_workspace_bytes(n_atoms, c.L, c.C, c.H)) : 0;
    w.bytes = o;
    return w;
}

e2f_status check_cfg(const e2f_attn_cfg* c) {
    if (!c) return E2F_ERR_INVALID_ARG;
    if (c->L < 0 || c->C <= 0 || c->H <= 0 || !(c->cutoff > 0.f) || !std::isfinite(c->cutoff))
        return E2F_ERR_INVALID_ARG;
    if (c->feat_dtype != E2F_F32 && c->feat_dtype != E2F_BF16) return E2F_ERR_UNSUPPORTED;
    if (c->m_max < -1) return E2F_ERR_INVALID_ARG;
    if (c->L > kMaxL || c->C % 16 != 0 || c->C > 256 || c->C % c->H != 0 || c->n_rbf < 2 || c->n_rbf > 32)
        return E2F_ERR_UNSUPPORTED;
    return E2F_OK;
}

}  // namespace

extern "C" const char* e2f_status_string(e2f_status s) {
    switch (s) {
        case E2F_OK: return "ok";
        case E2F_ERR_INVALID_ARG: return "invalid argument";
        case E2F_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case E2F_ERR_CAPACITY: return "output capacity too small";
        case E2F_ERR_ALIGNMENT: return "misaligned pointer";
        case E2F_ERR_TIMEOUT: return "device-side wait timed out";
        case E2F_ERR_CUDA: return "CUDA error";
        case E2F_ERR_NONFINITE: return "non-finite position";
        case E2F_ERR_STALE: return "reused cell lists are stale (an atom moved more than skin/2)";
    }
    return "unknown status";
}

extern "C" size_t e2f_attention_workspace_size(int64_t n_atoms, int64_t n_pairs, const e2f_attn_cfg* cfg) {
    (void)n_pairs;
    if (check_cfg(cfg) != E2F_OK || n_atoms < 0) return 0;
    return attn_layout(n_atoms, *cfg).bytes;
}

extern "C" e2f_status e2f_onfly_attention(const e2f_attn_cfg* cfg, const float* pos, int64_t n_atoms,
                                          const float* box_host, const int32_t* row_ptr, const int32_t* col,
                                          int64_t n_pairs, const void* x, const float* W_q, const float* W_k,
                                          const float* W_rad, const void* W_so2, float* out, void* workspace,
                                          size_t ws_bytes, void* stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    e2f_status st = check_cfg(cfg);
    if (st != E2F_OK) return st;
    if (n_atoms < 0 || n_atoms > INT32_MAX || n_pairs < 0 || n_pairs > INT32_MAX) return E2F_ERR_INVALID_ARG;
    if (n_atoms == 0) return E2F_OK;
    if (!pos || !row_ptr || (n_pairs > 0 && !col) || !x || !W_q || !W_k || !W_rad || !W_so2 || !out || !workspace)
        return E2F_ERR_INVALID_ARG;
    if (box_host) {
        for (int a = 0; a < 3; ++a)
            if (!(box_host[a] > 0.f) || !std::isfinite(box_host[a]) || cfg->cutoff > 0.5f * box_host[a])
                return E2F_ERR_INVALID_ARG;
    }
    if (reinterpret_cast<uintptr_t>(workspace) % 256 || reinterpret_cast<uintptr_t>(x) % 16 ||
        reinterpret_cast<uintptr_t>(W_so2) % 16 || reinterpret_cast<uintptr_t>(out) % 16 ||
        reinterpret_cast<uintptr_t>(W_rad) % 16)
        return E2F_ERR_ALIGNMENT;
    AttnWs L = attn_layout(n_atoms, *cfg);
    if (ws_bytes < L.bytes) return E2F_ERR_INVALID_ARG;
    char* ws = static_cast<char*>(workspace);

    AttnArgs a{};
    a.L = cfg->L; a.C = cfg->C; a.H = cfg->H; a.n_rbf = cfg->n_rbf; a.cutoff = cfg->cutoff;
    a.M = effective_mmax(cfg->L, cfg->m_max);
    a.bf16 = cfg->feat_dtype == E2F_BF16;
    a.n_atoms = (int)n_atoms; a.n_pairs = n_pairs;
    a.box.periodic = box_host != nullptr;
    if (box_host) {
        a.box.len = make_float3(box_host[0], box_host[1], box_host[2]);
        a.box.inv = make_float3(1.0f / box_host[0], 1.0f / box_host[1], 1.0f / box_host[2]);
    } else {
        a.box.len = a.box.inv = make_float3(0.f, 0.f, 0.f);
    }
    a.pos = pos; a.row_ptr = row_ptr; a.col = col; a.x = x;
    a.Wq = W_q; a.Wk = W_k; a.Wrad = W_rad; a.Wso2 = W_so2; a.out = out;
    a.status = reinterpret_cast<int*>(ws + L.o_status);
    a.q = reinterpret_cast<float*>(ws + L.o_q);
    a.k = reinterpret_cast<float*>(ws + L.o_k);
    a.Wt = L.tc ? nullptr : reinterpret_cast<float*>(ws + L.o_wt);
    E2F_CUDA_TRY(cudaMemsetAsync(a.status, 0, sizeof(int), stream));
    if (L.tc) {
        E2F_CUDA_TRY(run_attention_tc(a, ws + L.o_tc, stream));
    } else {
        E2F_CUDA_TRY(run_attention_simt(a, stream));
    }
    return E2F_OK;
}

extern "C" size_t e2f_attention_cells_skin_workspace_size(int64_t n_atoms, const float* box_host,
                                                          const e2f_attn_cfg* cfg, float skin) {
    if (check_cfg(cfg) != E2F_OK || n_atoms < 0 || !(skin >= 0.f) || !std::isfinite(skin)) return 0;
    if (box_host)
        for (int a = 0; a < 3; ++a)
            if (!(box_host[a] > 0.f) || !std::isfinite(box_host[a]) || cfg->cutoff > 0.5f * box_host[a]) return 0;
    return attn_layout(n_atoms, *cfg).bytes + align_up(cell_lists_bytes(n_atoms, box_host, cfg->cutoff, skin), 256);
}

extern "C" size_t e2f_attention_cells_workspace_size(int64_t n_atoms, const float* box_host,
                                                     const e2f_attn_cfg* cfg) {
    return e2f_attention_cells_skin_workspace_size(n_atoms, box_host, cfg, 0.f);
}

// Verlet-skin reuse: the parameters each workspace's cell lists were last
// sorted for (host side, keyed by the workspace address). A reuse call must
// match them; this catches a missing rebuild or a changed system without a
// device synchronisation.
struct SkinKey {
    int64_t n;
    float box[3], cutoff, skin;
    size_t cl_off;  // where the lists sit in the workspace (depends on cfg)
    bool periodic;
    bool operator==(const SkinKey& o) const {
        return n == o.n && periodic == o.periodic && cutoff == o.cutoff && skin == o.skin && cl_off == o.cl_off &&
               (!periodic || (box[0] == o.box[0] && box[1] == o.box[1] && box[2] == o.box[2]));
    }
};
static std::mutex g_skin_mu;
static std::unordered_map<const void*, SkinKey> g_skin_lists;
constexpr size_t kSkinTableMax = 4096;  // workspaces remembered; beyond it one entry is dropped

static e2f_status attention_cells(const e2f_attn_cfg* cfg, const float* pos, int64_t n_atoms, const float* box_host,
                                  float skin, bool rebuild, const void* x, const float* W_q, const float* W_k,
                                  const float* W_rad, const void* W_so2, float* out, void* workspace,
                                  size_t ws_bytes, void* stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    e2f_status st = check_cfg(cfg);
    if (st != E2F_OK) return st;
    if (n_atoms < 1 || n_atoms > INT32_MAX) return E2F_ERR_INVALID_ARG;
    if (!(skin >= 0.f) || !std::isfinite(skin) || (!rebuild && !(skin > 0.f))) return E2F_ERR_INVALID_ARG;
    if (!tc_supported(cfg->L, cfg->C, cfg->H, cfg->n_rbf, cfg->feat_dtype == E2F_BF16)) return E2F_ERR_UNSUPPORTED;
    if (!pos || !x || !W_q || !W_k || !W_rad || !W_so2 || !out || !workspace) return E2F_ERR_INVALID_ARG;
    if (box_host)
        for (int a = 0; a < 3; ++a)
            if (!(box_host[a] > 0.f) || !std::isfinite(box_host[a]) || cfg->cutoff > 0.5f * box_host[a])
                return E2F_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 || reinterpret_cast<uintptr_t>(x) % 16 ||
        reinterpret_cast<uintptr_t>(W_so2) % 16 || reinterpret_cast<uintptr_t>(out) % 16 ||
        reinterpret_cast<uintptr_t>(W_rad) % 16)
        return E2F_ERR_ALIGNMENT;
    AttnWs L = attn_layout(n_atoms, *cfg);
    const size_t cl_off = L.bytes;
    if (ws_bytes < cl_off + cell_lists_bytes(n_atoms, box_host, cfg->cutoff, skin)) return E2F_ERR_INVALID_ARG;
    char* ws = static_cast<char*>(workspace);
    SkinKey key{n_atoms, {0.f, 0.f, 0.f}, cfg->cutoff, skin, cl_off, box_host != nullptr};
    if (box_host) for (int a = 0; a < 3; ++a) key.box[a] = box_host[a];
    CellLists cl;
    if (rebuild) {
        {
            std::lock_guard<std::mutex> lk(g_skin_mu);
            g_skin_lists.erase(workspace);
        }
        E2F_CUDA_TRY(build_cell_lists(pos, (int)n_atoms, box_host, cfg->cutoff, ws + cl_off, &cl, stream, skin));
        if (skin > 0.f) {
            std::lock_guard<std::mutex> lk(g_skin_mu);
            if (g_skin_lists.size() >= kSkinTableMax) g_skin_lists.erase(g_skin_lists.begin());
            g_skin_lists[workspace] = key;
        }
    } else {
        {
            std::lock_guard<std::mutex> lk(g_skin_mu);
            auto it = g_skin_lists.find(workspace);
            if (it == g_skin_lists.end() || !(it->second == key)) return E2F_ERR_INVALID_ARG;
        }
        E2F_CUDA_TRY(refresh_cell_lists(pos, (int)n_atoms, box_host, cfg->cutoff, skin, ws + cl_off, &cl, stream));
    }

    AttnArgs a{};
    a.L = cfg->L; a.C = cfg->C; a.H = cfg->H; a.n_rbf = cfg->n_rbf; a.cutoff = cfg->cutoff;
    a.M = effective_mmax(cfg->L, cfg->m_max);
    a.bf16 = true;
    a.n_atoms = (int)n_atoms; a.n_pairs = 0;
    a.box.periodic = box_host != nullptr;
    if (box_host) {
        a.box.len = make_float3(box_host[0], box_host[1], box_host[2]);
        a.box.inv = make_float3(1.0f / box_host[0], 1.0f / box_host[1], 1.0f / box_host[2]);
    } else {
        a.box.len = a.box.inv = make_float3(0.f, 0.f, 0.f);
    }
    a.pos = pos; a.row_ptr = cl.rp; a.col = nullptr; a.x = x;
    a.Wq = W_q; a.Wk = W_k; a.Wrad = W_rad; a.Wso2 = W_so2; a.out = out;
    a.status = reinterpret_cast<int*>(ws + L.o_status);
    a.q = reinterpret_cast<float*>(ws + L.o_q);
    a.k = reinterpret_cast<float*>(ws + L.o_k);
    a.Wt = nullptr;
    E2F_CUDA_TRY(cudaMemsetAsync(a.status, 0, sizeof(int), stream));
    E2F_CUDA_TRY(run_attention_tc(a, ws + L.o_tc, stream, &cl));
    return E2F_OK;
}

extern "C" e2f_status e2f_onfly_attention_cells(const e2f_attn_cfg* cfg, const float* pos, int64_t n_atoms,
                                                const float* box_host, const void* x, const float* W_q,
                                                const float* W_k, const float* W_rad, const void* W_so2,
                                                float* out, void* workspace, size_t ws_bytes, void* stream) {
    return attention_cells(cfg, pos, n_atoms, box_host, 0.f, true, x, W_q, W_k, W_rad, W_so2, out, workspace,
                           ws_bytes, stream);
}

extern "C" e2f_status e2f_onfly_attention_cells_skin(const e2f_attn_cfg* cfg, const float* pos, int64_t n_atoms,
                                                     const float* box_host, float skin, int rebuild, const void* x,
                                                     const float* W_q, const float* W_k, const float* W_rad,
                                                     const void* W_so2, float* out, void* workspace,
                                                     size_t ws_bytes, void* stream) {
    return attention_cells(cfg, pos, n_atoms, box_host, skin, rebuild != 0, x, W_q, W_k, W_rad, W_so2, out,
                           workspace, ws_bytes, stream);
}

extern "C" e2f_status e2f_attention_status(void* workspace, size_t ws_bytes, void* stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    if (!workspace || ws_bytes < 256) return E2F_ERR_INVALID_ARG;
    int v = 0;
    E2F_CUDA_TRY(cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream));
    E2F_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(int), stream));
    E2F_CUDA_TRY(cudaStreamSynchronize(stream));
    E2F_CUDA_TRY(cudaGetLastError());
    return v == 0 ? E2F_OK : static_cast<e2f_status>(v);
}

extern "C" e2f_status e2f_edge_wigner_blocks(const float* r, int64_t n_edges, int L, float* out, float* frames,
                                             void* stream_) {
    if (L < 0 || L > kMaxL || n_edges < 0) return L > kMaxL ? E2F_ERR_UNSUPPORTED : E2F_ERR_INVALID_ARG;
    if (n_edges == 0) return E2F_OK;
    if (!r || !out) return E2F_ERR_INVALID_ARG;
    E2F_CUDA_TRY(run_edge_wigner(r, n_edges, L, out, frames, static_cast<cudaStream_t>(stream_)));
    return E2F_OK;
}

extern "C" int64_t e2f_launch_count(void) { return (int64_t)g_launches.load(); }

extern "C" int e2f_attention_uses_tensor_cores(const e2f_attn_cfg* cfg) {
    if (check_cfg(cfg) != E2F_OK) return 0;
    return tc_supported(cfg->L, cfg->C, cfg->H, cfg->n_rbf, cfg->feat_dtype == E2F_BF16) ? 1 : 0;
}

extern "C" void e2f_attention_set_kernel_events(void* start_event, void* stop_event) {
    set_tc_kernel_events(start_event, stop_event);
}

extern "C" void e2f_attention_set_debug(int max_ctas, int timers, int drop_arrive) {
    set_tc_debug(max_ctas, timers, drop_arrive);
}

namespace {

struct BwdWs {
    size_t o_status, o_q, o_k, o_wt, o_lse, o_gq, o_gk, o_beta, o_part, o_w16, o_ops, bytes;
};

BwdWs bwd_layout(int64_t n_atoms, int64_t n_pairs, const e2f_attn_cfg& c) {
    BwdWs w{};
    size_t o = 0;
    auto take = [&](size_t b) { size_t r = o; o = align_up(o + b, 256); return r; };
    w.o_status = take(256);  // first, as in the forward layout: e2f_attention_status reads it
    w.o_q = take(4 * (size_t)n_atoms * c.C);
    w.o_k = take(4 * (size_t)n_atoms * c.C);
    w.o_wt = take(4 * so2_total(c.L, c.C, effective_mmax(c.L, c.m_max)));
    w.o_lse = take(4 * (size_t)n_atoms * c.H);
    w.o_gq = take(4 * (size_t)n_atoms * c.C);
    w.o_gk = take(4 * (size_t)n_atoms * c.C);
    w.o_beta = take(4 * (size_t)n_pairs * c.H);
    const bool bf = c.feat_dtype == E2F_BF16;
    w.o_part = bf ? 0 : take(bwd_partial_bytes(c.L, c.C, effective_mmax(c.L, c.m_max)));
    w.o_w16 = bf ? take(4 * so2_total(c.L, c.C, effective_mmax(c.L, c.m_max))) : 0;
    w.o_ops = bf ? take(bwd_ops_bytes(n_pairs, c.L, c.C)) : 0;
    w.bytes = o;
    return w;
}

}  // namespace

extern "C" size_t e2f_attention_backward_workspace_size(int64_t n_atoms, int64_t n_pairs, const e2f_attn_cfg* cfg) {
    if (check_cfg(cfg) != E2F_OK || n_atoms < 0 || n_pairs < 0) return 0;
    return bwd_layout(n_atoms, n_pairs, *cfg).bytes;
}

extern "C" e2f_status e2f_onfly_attention_backward(const e2f_attn_cfg* cfg, const float* pos, int64_t n_atoms,
                                                   const float* box_host, const int32_t* row_ptr,
                                                   const int32_t* col, int64_t n_pairs, const void* x,
                                                   const float* W_q, const float* W_k, const float* W_rad,
                                                   const void* W_so2, const float* grad_out, float* grad_pos,
                                                   float* grad_x, float* grad_W_q, float* grad_W_k,
                                                   float* grad_W_rad, float* grad_W_so2, void* workspace,
                                                   size_t ws_bytes, void* stream_) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    e2f_status st = check_cfg(cfg);
    if (st != E2F_OK) return st;
    if (!bwd_supported(cfg->L, cfg->C, cfg->H, cfg->n_rbf)) return E2F_ERR_UNSUPPORTED;
    if (cfg->feat_dtype == E2F_BF16 && cfg->H > 32) return E2F_ERR_UNSUPPORTED;  // weight-gradient operand build
    if (n_atoms < 0 || n_atoms > INT32_MAX || n_pairs < 0 || n_pairs > INT32_MAX) return E2F_ERR_INVALID_ARG;
    if (n_atoms == 0) return E2F_OK;
    if (!pos || !row_ptr || (n_pairs > 0 && !col) || !x || !W_q || !W_k || !W_rad || !W_so2 || !grad_out ||
        !grad_pos || !grad_x || !grad_W_rad || !workspace)
        return E2F_ERR_INVALID_ARG;
    if (box_host) {
        for (int a = 0; a < 3; ++a)
            if (!(box_host[a] > 0.f) || !std::isfinite(box_host[a]) || cfg->cutoff > 0.5f * box_host[a])
                return E2F_ERR_INVALID_ARG;
    }
    if (reinterpret_cast<uintptr_t>(workspace) % 256 || reinterpret_cast<uintptr_t>(x) % 16 ||
        reinterpret_cast<uintptr_t>(W_so2) % 16 || reinterpret_cast<uintptr_t>(grad_out) % 16 ||
        reinterpret_cast<uintptr_t>(grad_x) % 16)
        return E2F_ERR_ALIGNMENT;
    const BwdWs L = bwd_layout(n_atoms, n_pairs, *cfg);
    if (ws_bytes < L.bytes) return E2F_ERR_INVALID_ARG;
    char* ws = static_cast<char*>(workspace);

    BwdArgs b{};
    AttnArgs& a = b.fwd;
    a.L = cfg->L; a.C = cfg->C; a.H = cfg->H; a.n_rbf = cfg->n_rbf; a.cutoff = cfg->cutoff;
    a.M = effective_mmax(cfg->L, cfg->m_max);
    a.bf16 = cfg->feat_dtype == E2F_BF16;
    a.n_atoms = (int)n_atoms; a.n_pairs = n_pairs;
    a.box.periodic = box_host != nullptr;
    if (box_host) {
        a.box.len = make_float3(box_host[0], box_host[1], box_host[2]);
        a.box.inv = make_float3(1.0f / box_host[0], 1.0f / box_host[1], 1.0f / box_host[2]);
    } else {
        a.box.len = a.box.inv = make_float3(0.f, 0.f, 0.f);
    }
    a.pos = pos; a.row_ptr = row_ptr; a.col = col; a.x = x;
    a.Wq = W_q; a.Wk = W_k; a.Wrad = W_rad; a.Wso2 = W_so2;
    a.q = reinterpret_cast<float*>(ws + L.o_q);
    a.k = reinterpret_cast<float*>(ws + L.o_k);
    a.Wt = reinterpret_cast<float*>(ws + L.o_wt);
    b.grad_out = grad_out;
    b.lse = reinterpret_cast<float*>(ws + L.o_lse);
    b.beta = reinterpret_cast<float*>(ws + L.o_beta);
    b.gq = reinterpret_cast<float*>(ws + L.o_gq);
    b.gk = reinterpret_cast<float*>(ws + L.o_gk);
    b.gpos = grad_pos; b.gx = grad_x; b.gWq = grad_W_q; b.gWk = grad_W_k; b.gWrad = grad_W_rad;
    b.gWso2 = grad_W_so2;
    b.gWpart = cfg->feat_dtype == E2F_BF16 ? nullptr : reinterpret_cast<float*>(ws + L.o_part);
    b.w16 = cfg->feat_dtype == E2F_BF16 ? ws + L.o_w16 : nullptr;
    b.ops = cfg->feat_dtype == E2F_BF16 ? ws + L.o_ops : nullptr;
    b.status = reinterpret_cast<int*>(ws + L.o_status);
    E2F_CUDA_TRY(cudaMemsetAsync(b.status, 0, sizeof(int), stream));
    E2F_CUDA_TRY(run_attention_bwd(b, stream));
    return E2F_OK;
}

extern "C" e2f_status e2f_attention_debug_timers(void* workspace, size_t ws_bytes, int64_t n_atoms,
                                                const e2f_attn_cfg* cfg, int64_t* host_out, int n_values,
                                                void* stream_) {
    if (!workspace || !host_out || !cfg || n_values < 0) return E2F_ERR_INVALID_ARG;
    AttnWs L = attn_layout(n_atoms, *cfg);
    if (!L.tc || ws_bytes < L.bytes) return E2F_ERR_UNSUPPORTED;
    const size_t n = std::min((size_t)n_values, kTcDebugBytes / 8);
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    E2F_CUDA_TRY(cudaMemcpyAsync(host_out, static_cast<char*>(workspace) + L.o_tc, n * 8, cudaMemcpyDeviceToHost,
                                 stream));
    E2F_CUDA_TRY(cudaStreamSynchronize(stream));
    return E2F_OK;
}
