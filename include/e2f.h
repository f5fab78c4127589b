/*
 * e2f.h - C ABI of libe2f.so: a GPU cell-list neighbour build and the
 * node-centric on-the-fly equivariant attention forward pass of E2Former-V2
 * ("E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
 * Memory", arXiv 2601.16622; summarised on gist.science, Technical Summary
 * sections 2.1 and 2.2, and in the abstract on fugumt.com).
 *
 * Conventions shared by every entry point
 *   - Device pointers point to memory of the current CUDA device; host
 *     pointers are read (or written) before the call returns.
 *   - The caller owns every buffer. The library allocates no device memory
 *     of its own; it works inside the caller's workspace. Per device it keeps
 *     only lazily set kernel attributes and the static scratch array of
 *     e2f_build_neighbors_noalloc (module memory).
 *   - Work is enqueued on `stream` (0 = legacy default stream) in stream
 *     order. Calls that return a host value (n_pairs_host) synchronise it.
 *   - Argument checks happen before any launch; a failed check launches
 *     nothing and leaves every output untouched. Unsupported shapes return
 *     E2F_ERR_UNSUPPORTED. There is no CPU fallback.
 *   - Irreducible features use the flat index k(l, m) = l*l + l + m,
 *     m = -l..l, with real spherical harmonics ordered so that degree 1 is
 *     proportional to (y, z, x); the channel index is innermost.
 */
#ifndef E2F_H
#define E2F_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    E2F_OK = 0,
    E2F_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad range      */
    E2F_ERR_UNSUPPORTED = 2,  /* shape or dtype the library does not handle */
    E2F_ERR_CAPACITY = 3,     /* output buffer too small (see n_pairs_host)  */
    E2F_ERR_ALIGNMENT = 4,    /* pointer not aligned as documented           */
    E2F_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out          */
    E2F_ERR_CUDA = 6,         /* a CUDA runtime call or launch failed        */
    E2F_ERR_NONFINITE = 7,    /* NaN/Inf in positions                        */
    E2F_ERR_STALE = 8         /* reused cell lists: an atom moved > skin/2   */
} e2f_status;

typedef enum { E2F_F32 = 0, E2F_BF16 = 1 } e2f_dtype;

/* Layer shape. L = highest degree (0..4); C = channels (multiple of 16,
 * 16..256); H = attention heads (divides C); n_rbf = radial basis size
 * (2..32); cutoff in the positions' length unit; feat_dtype = storage type of
 * x and W_so2 (E2F_F32 or E2F_BF16). Arithmetic accumulates in fp32. */
typedef struct {
    int L;
    int C;
    int H;
    int n_rbf;
    float cutoff;
    e2f_dtype feat_dtype;
    /* SO(2) truncation: the maps act on |m| <= M only, M = m_max (0 <= m_max
     * < L), or M = L when m_max < 0 or m_max >= L (the full layer). Rows with
     * |m| > M get no message (as if A(m), B(m) were zero); W_so2 holds the
     * blocks m <= M only. */
    int m_max;
} e2f_attn_cfg;

/* Human-readable name of a status code (static string, never NULL). */
const char* e2f_status_string(e2f_status s);

/* ------------------------------------------------------------------------
 * Neighbour list (cell list).
 *
 * The pages iterate over "j in N(i)" (gist.science Technical Summary 2.2)
 * without saying how N(i) is found. This builds it with a linked-cell grid:
 * j is a neighbour of i iff j != i, both lie in the same graph, and the
 * minimum-image distance passes this exact fp32 test (round-to-nearest, no
 * fused multiply-add):
 *     dx = x_j - x_i;  periodic: dx -= box * rint(dx * (1/box))   per axis
 *     d2 = (dx*dx + dy*dy) + dz*dz;   keep d2 < cutoff*cutoff
 * Output is CSR: row_ptr[N+1], col[E]; rows in atom order, columns
 * ascending within a row, self excluded, every pair listed in both
 * directions.
 *
 *   pos        device, float [N*3] (x, y, z per atom), finite. Periodic
 *              positions may lie outside the box; the image is implied.
 *   n_atoms    N >= 0 (N = 0 gives row_ptr = {0} and E = 0).
 *   box_host   host, float[3] orthorhombic box lengths, or NULL for open
 *              boundaries. Requires cutoff <= min(box)/2.
 *   cutoff     > 0.
 *   graph_ptr  device, int32 [n_graphs+1], non-decreasing from 0 to N; or
 *              NULL (all atoms form one graph; n_graphs ignored).
 *   row_ptr    device, int32 [N+1], written.
 *   col        device, int32 [col_capacity], written (first E entries).
 *   n_pairs_host  host, written with E on success and on E2F_ERR_CAPACITY
 *              (then row_ptr holds the offsets and col is not written;
 *              grow col and call again). On E2F_ERR_NONFINITE or a bad
 *              graph_ptr (E2F_ERR_INVALID_ARG) row_ptr is unspecified.
 *   workspace  device, >= e2f_neighbors_workspace_size(...) bytes,
 *              256-byte aligned. Contents need no initialisation.
 * Synchronises `stream` (E is returned to the host). E must fit in int32.
 * ---------------------------------------------------------------------- */
size_t e2f_neighbors_workspace_size(int64_t n_atoms, const float* box_host,
                                    float cutoff, int32_t n_graphs);

e2f_status e2f_build_neighbors(const float* pos, int64_t n_atoms,
                               const float* box_host, float cutoff,
                               const int32_t* graph_ptr, int32_t n_graphs,
                               int32_t* row_ptr, int32_t* col,
                               int64_t col_capacity, int64_t* n_pairs_host,
                               void* workspace, size_t ws_bytes,
                               void* stream);

/* The same list for the destination rows 0 .. n_rows-1 only: rows n_rows ..
 * N-1 are empty (row_ptr constant there), while every atom remains a
 * candidate neighbour of the query rows. The node-centric layer needs, for
 * each destination node, only its own neighbours (gist.science Technical
 * Summary 2.2, Eq. 6), so a rank of a spatial decomposition that holds its
 * owned atoms first and their halo after needs the rows of its owned atoms
 * only; searching the halo atoms' rows would be wasted work. Arguments,
 * outputs, checks and synchronisation as for e2f_build_neighbors;
 * 0 <= n_rows <= n_atoms (E2F_ERR_INVALID_ARG otherwise). The rows
 * 0 .. n_rows-1 equal those of e2f_build_neighbors on the same atoms. */
e2f_status e2f_build_neighbors_rows(const float* pos, int64_t n_atoms,
                                    int64_t n_rows, const float* box_host,
                                    float cutoff, const int32_t* graph_ptr,
                                    int32_t n_graphs, int32_t* row_ptr,
                                    int32_t* col, int64_t col_capacity,
                                    int64_t* n_pairs_host, void* workspace,
                                    size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Neighbour list without a caller workspace. The pages have no counterpart
 * of this call: it exists for callers that cannot allocate device memory
 * when they need the list (an allocator of another runtime owns the heap,
 * or cudaMalloc's device-wide synchronisation is not acceptable).
 *
 * Same arguments, outputs, checks and results as e2f_build_neighbors, minus
 * workspace/ws_bytes: the scratch is a static device array of this library
 * of E2F_NOALLOC_SCRATCH_BYTES (16 MiB) per device, enough for about 390k
 * atoms with open boundaries or 500k in a periodic box at a 6 A cutoff.
 * The call allocates no device memory.
 *   Returns E2F_ERR_UNSUPPORTED, before any launch, when
 *   e2f_neighbors_workspace_size(...) exceeds E2F_NOALLOC_SCRATCH_BYTES;
 *   E2F_ERR_CUDA if the scratch address cannot be looked up.
 * The scratch is shared: calls that overlap on one device (other threads,
 * other streams, or a call enqueued while an earlier one's kernels still
 * run) race on it and give undefined results; serialise them. Every call
 * looks up the array's device address in the context current on the
 * calling thread, so a device reset or another context on the same device
 * gets its own copy; the first call in a context may load the module, so
 * make it before any stream capture starts there. The call synchronises
 * `stream` once, to read the pair count, and returns with the column-fill
 * kernel still queued on `stream`; that kernel reads the scratch, so the
 * scratch is free again only once it has run: enqueue the next call on the
 * same stream, or synchronise `stream` first.
 * ---------------------------------------------------------------------- */
#define E2F_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

e2f_status e2f_build_neighbors_noalloc(const float* pos, int64_t n_atoms,
                                       const float* box_host, float cutoff,
                                       const int32_t* graph_ptr,
                                       int32_t n_graphs, int32_t* row_ptr,
                                       int32_t* col, int64_t col_capacity,
                                       int64_t* n_pairs_host, void* stream);

/* ------------------------------------------------------------------------
 * On-the-fly equivariant attention, forward (gist.science Technical
 * Summary 2.1 EAAS: Lemma 4.1 and the re-indexing rule Eq. 13; 2.2:
 * node-centric factorisation Eq. 6, streaming reduction over j in N(i),
 * online softmax, no N x K x H x D tensor in HBM).
 *
 * For each node i and neighbour j (r = mic(x_j - x_i), d = |r|):
 *   rho_k(d) = u(d) exp(-((d - k rc/(n_rbf-1)) / (rc/(n_rbf-1)))^2),
 *              u(d) = (cos(pi d/rc) + 1)/2;   [g_v | g_a] = rho W_rad
 *   h        = g_v[l, c] * x_j[l, m, c]
 *   v_ij     = D(R)^T SO2(D(R) h),  R r = |r| z,  D = real Wigner-D blocks
 *              (Y_l(R v) = D^l(R) Y_l(v)); SO2 per |m| block:
 *              o[l3,+m] = sum_l1 A(m)[l3,l1] h[l1,+m] - B(m)[l3,l1] h[l1,-m]
 *              o[l3,-m] = sum_l1 B(m)[l3,l1] h[l1,+m] + A(m)[l3,l1] h[l1,-m]
 *   a_ij^h   = g_a^h <q_i^h, k_j^h> / sqrt(C/H),  q = W_q x[l=0], k = W_k x[l=0]
 *   out_i[l,m,c] = sum_j softmax_j(a_ij^{h(c)}) v_ij[l,m,c],  h(c) = c/(C/H);
 *   out_i = 0 when N(i) is empty.
 *
 *   cfg        host; shape and dtype (see e2f_attn_cfg).
 *   pos        device, float [N*3]; box_host as for the neighbour build.
 *   row_ptr, col  device CSR as produced by e2f_build_neighbors (any CSR
 *              with rows in atom order is accepted; col entries in [0, N)).
 *   n_pairs    E = row_ptr[N].
 *   x          device, [N, (L+1)^2, C] of feat_dtype, 16-byte aligned.
 *   W_q, W_k   device, float [C, C] row-major: q[c] = sum_c' W_q[c,c'] x[0,c'].
 *   W_rad      device, float [n_rbf, (L+1)C + H] row-major; column l*C + c
 *              is g_v[l, c], column (L+1)C + h is g_a^h. 16-byte aligned.
 *   W_so2      device, feat_dtype, packed: A(0), then A(m), B(m) for
 *              m = 1..M (M = L unless cfg->m_max truncates); block m is a
 *              row-major square matrix of side (L+1-m)C indexed
 *              [(l3, c_out), (l1, c_in)], l3, l1 = m..L. 85*C*C values at
 *              L = 4 (full). 16-byte aligned.
 *   out        device, float [N, (L+1)^2, C], written.
 *   workspace  device, >= e2f_attention_workspace_size(...) bytes, 256-byte
 *              aligned, contents need no initialisation. Holds the
 *              repacked weights, per-node Q/K and softmax statistics and a
 *              device status word; it must not be shared by calls in flight.
 * Launch shape: the tensor-core kernel runs one persistent CTA per SM
 * (e2f_attention_set_debug can cap that count, which lets tests give each
 * CTA many tiles on small systems).
 * Asynchronous: returns after enqueueing. Device-side failures (a bounded
 * wait that ran out) are recorded in the workspace status word; read it
 * with e2f_attention_status.
 * ---------------------------------------------------------------------- */
size_t e2f_attention_workspace_size(int64_t n_atoms, int64_t n_pairs,
                                    const e2f_attn_cfg* cfg);

e2f_status e2f_onfly_attention(const e2f_attn_cfg* cfg, const float* pos,
                               int64_t n_atoms, const float* box_host,
                               const int32_t* row_ptr, const int32_t* col,
                               int64_t n_pairs, const void* x,
                               const float* W_q, const float* W_k,
                               const float* W_rad, const void* W_so2,
                               float* out, void* workspace, size_t ws_bytes,
                               void* stream);

/* 1 when e2f_onfly_attention runs this shape on the tcgen05 tensor-core
 * kernel (bf16 features, L >= 1, C = 64 or a multiple of 128 up to 256, H <= 16 and
 * a multiple of 4), 0 when it runs the fp32 CUDA-core kernel. */
int e2f_attention_uses_tensor_cores(const e2f_attn_cfg* cfg);

/* Profiling aid (no counterpart in the pages). start_event and stop_event
 * are cudaEvent_t handles created by the caller. While both are non-NULL,
 * every e2f_onfly_attention call that runs the tensor-core kernel records
 * start_event on its stream just before that kernel and stop_event just
 * after, so cudaEventElapsedTime gives the main kernel alone (without the
 * O(N) pre-passes). NULL, NULL turns it off. One process-wide setting: not
 * for concurrent calls from several threads. */
void e2f_attention_set_kernel_events(void* start_event, void* stop_event);

/* Debug and test controls of the tensor-core kernel (no counterpart in the
 * pages). One process-wide setting, read when a call is enqueued; not for
 * concurrent calls from several threads. All zero (the default) is the
 * product behaviour.
 *   max_ctas     > 0: at most this many persistent CTAs (fewer, longer CTAs).
 *   timers       != 0: record the role cycle counters (e2f_attention_debug_timers).
 *   drop_arrive  != 0: CTA 0 withholds one producer arrival on its first tile,
 *                so its bounded waits run out (about 2 s): the CTA records
 *                E2F_ERR_TIMEOUT in the workspace status word, drains what it
 *                issued and returns; the other CTAs finish normally. Used to
 *                test the timeout path; the output of such a call is invalid. */
void e2f_attention_set_debug(int max_ctas, int timers, int drop_arrive);

/* Diagnostics of the tensor-core kernel. When timers are on
 * (e2f_attention_set_debug), each persistent CTA records clock64
 * cycle counts of its warp roles into the workspace: per CTA 32 int64 values,
 * [0] producer wait for a free tile buffer, [1] producer total, [2] TMA wait
 * for features, [3] TMA wait for a free ring stage, [4] TMA total, [5] MMA
 * wait for a free TMEM group, [6] MMA wait for a full stage, [7] MMA total,
 * [8] epilogue wait for tile data, [9] epilogue wait for accumulators,
 * [10] epilogue total, [11] producer per-edge setup, [12] producer feature
 * rotation, [13] tiles, [14..21] sub-steps of the per-edge setup (one
 * thread's view: node search, geometry, Wigner blocks, their stores, radial
 * basis, logits, barrier, value gate), [22] epilogue rotate-back; the rest
 * is zero. Copies the first n_values counters to host_out
 * (synchronises `stream`). No counterpart in the paper: a profiling aid. */
e2f_status e2f_attention_debug_timers(void* workspace, size_t ws_bytes, int64_t n_atoms,
                                      const e2f_attn_cfg* cfg, int64_t* host_out, int n_values,
                                      void* stream);

/* ------------------------------------------------------------------------
 * On-the-fly equivariant attention with the cell-list traversal fused in
 * (no neighbour list in memory): the same layer as e2f_onfly_attention,
 * but the kernels find each node's neighbours themselves from a cell list
 * of the positions (the neighbour build's grid, buckets ordered by atom
 * index), so no E-sized array (col) is written or read. Only O(N) data is
 * kept: the cell lists and per-node edge offsets. Nodes are processed in
 * cell order. The neighbour set is the exact fp32 predicate of
 * e2f_build_neighbors (cutoff = cfg->cutoff); the order of the edges of a
 * node differs from the CSR call, so sums may differ in the last bits.
 *
 * Periodic boxes (box_host non-NULL, cutoff <= min(box)/2) or open
 * boundaries (box_host NULL: the neighbour build's hashed cells; cells
 * that hash to one bucket are visited once). The tensor-core
 * configurations (e2f_attention_uses_tensor_cores) only; otherwise
 * E2F_ERR_UNSUPPORTED. One system (no graph batching).
 * Arguments as for e2f_onfly_attention without row_ptr, col, n_pairs;
 * workspace >= e2f_attention_cells_workspace_size(...) bytes, 256-byte
 * aligned. Asynchronous (no host synchronisation); non-finite positions
 * are reported through e2f_attention_status as E2F_ERR_NONFINITE.
 * ---------------------------------------------------------------------- */
size_t e2f_attention_cells_workspace_size(int64_t n_atoms, const float* box_host,
                                          const e2f_attn_cfg* cfg);

e2f_status e2f_onfly_attention_cells(const e2f_attn_cfg* cfg, const float* pos,
                                     int64_t n_atoms, const float* box_host,
                                     const void* x, const float* W_q,
                                     const float* W_k, const float* W_rad,
                                     const void* W_so2, float* out,
                                     void* workspace, size_t ws_bytes,
                                     void* stream);

/* ------------------------------------------------------------------------
 * The same fused call with Verlet-skin reuse of the cell lists across
 * molecular-dynamics steps (the layer's conservative variant drives MD,
 * gist.science Technical Summary 2.2: positions move a little per step, so
 * the sort of the atoms into cells need not be redone every step).
 * skin >= 0 (length units of pos).
 *
 *   rebuild != 0  sort the atoms into cells at least cutoff + skin wide and
 *                 keep their positions in the workspace (the reference
 *                 positions); then the layer as e2f_onfly_attention_cells.
 *   rebuild == 0  (skin > 0, else E2F_ERR_INVALID_ARG) reuse the sort held
 *                 in `workspace` from the last rebuild call on it, which
 *                 must have had the same n_atoms, box, cfg and skin: the
 *                 library records these per workspace address at each
 *                 successful rebuild and returns E2F_ERR_INVALID_ARG, before
 *                 any launch, when they differ or no rebuild is recorded
 *                 (host-side check by address: a buffer that is freed and
 *                 allocated again at the same address is not told apart,
 *                 so the first call on any new buffer must rebuild; the
 *                 contents must still be the ones that rebuild wrote; at
 *                 most 4096 workspaces are remembered, and a reuse call on
 *                 a forgotten one returns E2F_ERR_INVALID_ARG):
 *                 each atom's slot takes its current position and the
 *                 neighbours of an atom are searched around its reference
 *                 cell. Exact while every atom lies within skin/2 of its
 *                 reference position (minimum image): then every pair within
 *                 the cutoff now was within cutoff + skin then, so it sits in
 *                 the stencil searched. Otherwise e2f_attention_status
 *                 reports E2F_ERR_STALE, `out` is unspecified, and the caller
 *                 repeats the call with rebuild != 0.
 *
 * The neighbour set and the pair test are those of e2f_onfly_attention_cells
 * (cutoff = cfg->cutoff, not cutoff + skin); the edge order differs with the
 * cell size, so sums may differ in the last bits. skin == 0 with rebuild != 0
 * is e2f_onfly_attention_cells. workspace >=
 * e2f_attention_cells_skin_workspace_size(...) bytes (16 bytes per atom
 * more than without a skin), 256-byte aligned. Asynchronous.
 * ---------------------------------------------------------------------- */
size_t e2f_attention_cells_skin_workspace_size(int64_t n_atoms,
                                               const float* box_host,
                                               const e2f_attn_cfg* cfg,
                                               float skin);

e2f_status e2f_onfly_attention_cells_skin(const e2f_attn_cfg* cfg,
                                          const float* pos, int64_t n_atoms,
                                          const float* box_host, float skin,
                                          int rebuild, const void* x,
                                          const float* W_q, const float* W_k,
                                          const float* W_rad,
                                          const void* W_so2, float* out,
                                          void* workspace, size_t ws_bytes,
                                          void* stream);

/* ------------------------------------------------------------------------
 * Backward of the on-the-fly equivariant attention: the gradients of a
 * scalar loss with respect to every input of e2f_onfly_attention, given
 * grad_out = dLoss/dout. The pages' conservative variant takes forces as
 * the negative position gradient of the energy (gist.science Technical
 * Summary 2.2; the molecular-dynamics experiments), which this provides
 * (grad_pos); the weight gradients serve training. The pages print no
 * backward formulas: the call differentiates exactly the layer documented
 * above (same neighbour list, periodic image shifts held fixed) and
 * recomputes every per-edge quantity on chip, as the forward does; the
 * only O(E) scratch is one float per edge and head.
 *
 *   Arguments cfg .. W_so2 as for e2f_onfly_attention (same CSR, which
 *   need not be symmetric).
 *   grad_out    device, float [N, (L+1)^2, C].
 *   grad_pos    device, float [N*3], written.
 *   grad_x      device, float [N, (L+1)^2, C], written (fp32 for either
 *               feat_dtype).
 *   grad_W_q, grad_W_k   device, float [C, C], written; either may be
 *               NULL (not computed).
 *   grad_W_rad  device, float [n_rbf, (L+1)C + H], written.
 *   grad_W_so2  device, float, packed like W_so2 (truncation included),
 *               written; NULL skips it. With fp32 storage its kernel sweeps
 *               all edges per 64 x 64 tile of the SO(2) blocks. With bf16
 *               storage each edge's two operand rows (the rotated, gated
 *               features and the softmax-weighted rotated upstream
 *               gradient) are built once per chunk of 131,072 edges in the
 *               workspace, and each block's gradient is a GEMM over the
 *               chunk's edges, run by cuBLAS (loaded at run time; absent
 *               cuBLAS gives E2F_ERR_CUDA). One cuBLAS handle serves each
 *               CUDA context, so calls from several host threads at once
 *               on one context must be serialised by the caller.
 *   workspace   device, >= e2f_attention_backward_workspace_size(...)
 *               bytes, 256-byte aligned. Its status word (a bounded
 *               device-side wait that ran out: E2F_ERR_TIMEOUT) is read
 *               with e2f_attention_status, as for the forward.
 * Arithmetic: with fp32 storage, fp32 on CUDA cores throughout. With bf16
 * storage, the SO(2) maps and their transposes run on tensor cores
 * (mma.sync), and the SO(2) weight-gradient GEMMs on cuBLAS; all take fp16
 * operands with fp32 accumulation (about 3e-4 relative error against an
 * exact evaluation);
 * the rest stays fp32. Gradients that sum over edges use fp32 atomics, so
 * their last bits may differ between runs; grad_W_so2, grad_W_q and
 * grad_W_k are deterministic (the weight-gradient GEMMs run chunk after
 * chunk into the output). Shapes: those of e2f_onfly_attention with H
 * dividing 256 (at most 32 heads with bf16 storage) and the kernels' shared
 * memory within 227 KB (L = 4 allows C <= 128); otherwise
 * E2F_ERR_UNSUPPORTED. Asynchronous.
 * ---------------------------------------------------------------------- */
size_t e2f_attention_backward_workspace_size(int64_t n_atoms, int64_t n_pairs,
                                             const e2f_attn_cfg* cfg);

e2f_status e2f_onfly_attention_backward(const e2f_attn_cfg* cfg, const float* pos,
                                        int64_t n_atoms, const float* box_host,
                                        const int32_t* row_ptr, const int32_t* col,
                                        int64_t n_pairs, const void* x,
                                        const float* W_q, const float* W_k,
                                        const float* W_rad, const void* W_so2,
                                        const float* grad_out, float* grad_pos,
                                        float* grad_x, float* grad_W_q,
                                        float* grad_W_k, float* grad_W_rad,
                                        float* grad_W_so2, void* workspace,
                                        size_t ws_bytes, void* stream);

/* Synchronises `stream` and returns the device status recorded by the last
 * e2f_onfly_attention call on this workspace (E2F_OK or E2F_ERR_TIMEOUT);
 * each call clears the word when it starts. */
e2f_status e2f_attention_status(void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Edge-frame Wigner-D blocks, exposed for testing the rotation step alone
 * (gist.science Technical Summary 2.1, "SO(3) -> SO(2) change of basis").
 * For each unit-free direction r[e] (device, float [E*3], non-zero) writes
 * the blocks D^l(R_e), l = 0..L, R_e the rotation the attention kernels use
 * (R_e r = |r| z), row-major and concatenated: out[e*S + off(l) + a*(2l+1) + b]
 * with off(l) = sum_{l'<l} (2l'+1)^2, S = off(L+1). Also writes R_e itself
 * to frames[e*9 ...] (row-major) when frames is not NULL. Asynchronous.
 * ---------------------------------------------------------------------- */
e2f_status e2f_edge_wigner_blocks(const float* r, int64_t n_edges, int L,
                                  float* out, float* frames, void* stream);

/* Number of kernels this library has launched in this process (all
 * devices, all entry points); lets a caller count launches in a region. */
int64_t e2f_launch_count(void);

/* ------------------------------------------------------------------------
 * Wigner-6j node-level convolution: the E2Former attention variant whose
 * edge tensor product is moved onto the nodes (fugumt abstract page: EAAS
 * starts from this convolution, which takes the work from O(|E|) to O(|V|);
 * gist.science Technical Summary 3: EAAS joins Wigner-6j re-coupling with the
 * SO(2) alignment). The pages print no formula. The layer computed here,
 * open boundaries, r_ij = x_j - x_i:
 *   S^l_m(r) = sqrt(4 pi/(2l+1)) |r|^l Y_lm(r/|r|)    regular solid harmonics
 *              in the real basis of the main layer (S^0 = 1, S^1 = (y, z, x))
 *   v_ij[l3,m3,c] = sum over paths (l1,l2,l3) of w_path[p][c]
 *              sum_{m1,m2} Q^{l1l2l3}[m1,m2,m3] x_j[l1,m1,c] S^l2_m2(r_ij)
 *   a_ij^h   = g_a^h <q_i^h, k_j^h> / sqrt(C/H),  g_a = rho(|r_ij|) W_rad,
 *              rho and q, k as for e2f_onfly_attention
 *   out_i[l,m,c] = sum_j softmax_j(a_ij^{h(c)}) v_ij[l,m,c]; 0 if N(i) is empty
 * Q^{l1l2l3} is the real coupling tensor: with the unitary U_l taking the
 * complex harmonics (Condon-Shortley phase) to the real ones (none),
 *   Q[m1,m2,m3] = part of sum U3[m3,mu3] conj(U1[m1,mu1]) conj(U2[m2,mu2])
 *                 <l1 mu1 l2 mu2 | l3 mu3>,
 * the real part when l1+l2+l3 is even, the imaginary part when it is odd.
 * Paths, packed in this order: l1 = 0..L, then l3 = 0..L, then
 * l2 = |l1-l3| .. min(l1+l3, Lf); e2f_sixj_n_paths gives their count.
 *
 * The library never forms an edge tensor product: it expands S^l2(r_ij)
 * around each graph's mean position o (addition theorem of solid
 * harmonics), forms [x_j (x) S^lam(x_j - o)]^k per node, sums those with the
 * softmax weights over the edges, and re-couples with S^mu(o - x_i) per node
 * through the 6j symbols. The expansion's terms grow as (graph radius /
 * neighbour distance)^Lf while their sum does not, so the node products,
 * their sums and the tables are held in fp64 (inputs, logits and output are
 * fp32). The cost per atom grows with the graph's spread, not its size: the
 * layer is meant for molecules, not for extended systems (which also have no
 * single origin under periodic images).
 *
 *   cfg        host; L (0..4), Lf (0..2L, highest l2), C (1..256), H
 *              (1..32, divides C), n_rbf (2..32), cutoff > 0.
 *   pos        device, float [N*3]; open boundaries.
 *   graph_ptr  device, int32 [n_graphs+1] as for e2f_build_neighbors, or
 *              NULL (one graph). Every CSR pair must join two atoms of one
 *              graph (as e2f_build_neighbors lists them).
 *   row_ptr, col  device CSR, rows in atom order, col entries in [0, N).
 *   x          device, float [N, (L+1)^2, C].
 *   W_q, W_k   device, float [C, C] row-major (as for e2f_onfly_attention).
 *   W_rad      device, float [n_rbf, H] row-major: g_a = rho W_rad.
 *   w_path     device, float [n_paths, C].
 *   out        device, float [N, (L+1)^2, C], written.
 *   workspace  device, >= e2f_sixj_workspace_size(...) bytes, 256-byte
 *              aligned (0 from the size query means the shape is not
 *              supported). Holds the coupling tables and, per atom, the node
 *              products and their sums: 16 Z C + 8 C + 24 bytes, Z the number
 *              of node product components that reach the output (895 at
 *              L = 4, Lf = 8; 454 at L = 4, Lf = 4).
 * Errors: E2F_ERR_INVALID_ARG (null pointer, negative size, workspace too
 * small), E2F_ERR_UNSUPPORTED (shape outside the limits), E2F_ERR_ALIGNMENT,
 * E2F_ERR_CUDA. The coupling tables are built on the host the first time a
 * (L, Lf) is used and kept for the process; every call copies them from
 * that pageable host memory into the workspace on `stream` (the driver
 * stages such a copy before the call returns), so the call cannot be
 * captured into a CUDA graph. Otherwise asynchronous.
 * ---------------------------------------------------------------------- */
typedef struct {
    int L;
    int Lf;
    int C;
    int H;
    int n_rbf;
    float cutoff;
} e2f_sixj_cfg;

int e2f_sixj_n_paths(int L, int Lf);

size_t e2f_sixj_workspace_size(int64_t n_atoms, const e2f_sixj_cfg* cfg);

e2f_status e2f_sixj_attention(const e2f_sixj_cfg* cfg, const float* pos, int64_t n_atoms,
                              const int32_t* graph_ptr, int32_t n_graphs,
                              const int32_t* row_ptr, const int32_t* col,
                              int64_t n_pairs, const float* x, const float* W_q,
                              const float* W_k, const float* W_rad,
                              const float* w_path, float* out, void* workspace,
                              size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* E2F_H */
