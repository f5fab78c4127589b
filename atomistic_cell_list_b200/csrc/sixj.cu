// The Wigner-6j node-level convolution: an attention layer whose value is
// the tensor product of the neighbour's features with the regular solid
// harmonics of r_ij, evaluated on the nodes instead of the edges (fugumt
// abstract page: EAAS starts from the E2Former Wigner-6j convolution, which
// moves the work from edges to nodes; gist.science, Technical Summary 3:
// EAAS joins that re-coupling with the SO(2) axis alignment).
//
// With an origin o per graph, a_j = x_j - o and b_i = o - x_i, so
// r_ij = a_j + b_i, and the addition theorem of regular solid harmonics gives
//     S^l2(r_ij) = sum_lam sqrt(binom(2 l2, 2 lam)) [S^lam(a_j) (x) S^mu(b_i)]^l2,
// mu = l2 - lam. Re-coupling
//     [x^l1 (x) [S^lam (x) S^mu]^l2]^l3 = sum_k c_k [[x^l1 (x) S^lam]^k (x) S^mu]^l3,
// where c_k is the 6j symbol {l1 lam k; mu l3 l2} times sqrt((2k+1)(2 l2+1))
// and the phases of the real coupling tensors, splits the layer into
//     z_j   = [x_j^l1 (x) S^lam(a_j)]^k                   per node (k_sixj_node)
//     Z_i   = sum_j softmax_j(a_ij) z_j                    scalar weights per edge (k_sixj_agg)
//     out_i = sum w sqrt(binom) c_k [Z_i (x) S^mu(b_i)]^l3  per node (k_sixj_out)
// The library finds c_k by projecting one coupling scheme onto the other
// (the schemes' tensors are orthogonal, each of squared norm 2 l3 + 1), and
// checks that the projections rebuild the first scheme exactly.
#include <algorithm>
#include <cmath>
#include <complex>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include "common.cuh"
#include "e2f.h"

namespace e2f {
namespace sixj {

constexpr int kMaxLf = 2 * kMaxL;  // kMaxL = 4, the library's highest feature degree
constexpr int kMaxH = 32;
constexpr int kMaxRbf = 32;
constexpr int kAggE = 32;  // edges per aggregation chunk

// ---------------------------------------------------------------------------
// Host: Clebsch-Gordan coefficients and the real coupling tensors
// ---------------------------------------------------------------------------
using ld = long double;

ld fact(int n) {
    static const std::vector<ld> t = [] {
        std::vector<ld> v(64, 1.0L);
        for (int i = 1; i < 64; ++i) v[i] = v[i - 1] * (ld)i;
        return v;
    }();
    return t[n];
}

// <j1 m1 j2 m2 | J M> with the Condon-Shortley phase (Racah's sum)
ld clebsch(int j1, int m1, int j2, int m2, int J, int M) {
    if (m1 + m2 != M || std::abs(m1) > j1 || std::abs(m2) > j2 || std::abs(M) > J) return 0.0L;
    if (J < std::abs(j1 - j2) || J > j1 + j2) return 0.0L;
    const ld pre = std::sqrt((ld)(2 * J + 1) * fact(J + j1 - j2) * fact(J - j1 + j2) * fact(j1 + j2 - J) /
                             fact(j1 + j2 + J + 1) * fact(J + M) * fact(J - M) * fact(j1 - m1) * fact(j1 + m1) *
                             fact(j2 - m2) * fact(j2 + m2));
    ld s = 0.0L;
    for (int k = 0; k <= j1 + j2 - J; ++k) {
        const int a[6] = {k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k};
        bool ok = true;
        ld den = 1.0L;
        for (int q = 0; q < 6; ++q) {
            if (a[q] < 0) { ok = false; break; }
            den *= fact(a[q]);
        }
        if (ok) s += ((k & 1) ? -1.0L : 1.0L) / den;
    }
    return pre * s;
}

// U[m][mu] (row-major, indices offset by l): the library's real harmonic m
// (no Condon-Shortley phase) as a combination of complex harmonics mu (with
// that phase): for m > 0, Y_m = ((-1)^m Y^c_m + Y^c_-m)/sqrt2 and
// Y_-m = i (Y^c_-m - (-1)^m Y^c_m)/sqrt2; Y_0 = Y^c_0.
std::vector<std::complex<ld>> real_from_complex(int l) {
    const int n = 2 * l + 1;
    std::vector<std::complex<ld>> U((size_t)n * n, 0.0L);
    const ld h = 1.0L / std::sqrt(2.0L);
    U[(size_t)l * n + l] = 1.0L;
    for (int m = 1; m <= l; ++m) {
        const ld sg = (m & 1) ? -1.0L : 1.0L;
        U[(size_t)(l + m) * n + (l + m)] = sg * h;
        U[(size_t)(l + m) * n + (l - m)] = h;
        U[(size_t)(l - m) * n + (l - m)] = std::complex<ld>(0.0L, h);
        U[(size_t)(l - m) * n + (l + m)] = std::complex<ld>(0.0L, -sg * h);
    }
    return U;
}

// The real coupling tensor Q[a][b][c] of degrees (l1, l2, l3), dense:
// Q = sum U3[c][i] conj(U1[a][j]) conj(U2[b][k]) <l1 j l2 k | l3 i>, whose
// real part (l1+l2+l3 even) or imaginary part (odd) is kept; the other part
// is zero.
const std::vector<double>& coupling(int l1, int l2, int l3) {
    static std::mutex mu;
    static std::map<std::tuple<int, int, int>, std::vector<double>> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_tuple(l1, l2, l3);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    const int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
    const auto U1 = real_from_complex(l1), U2 = real_from_complex(l2), U3 = real_from_complex(l3);
    std::vector<std::complex<ld>> cgt((size_t)n1 * n2 * n3, 0.0L);  // [j][k][i] in complex indices
    for (int j = 0; j < n1; ++j)
        for (int k = 0; k < n2; ++k) {
            const int i = (j - l1) + (k - l2) + l3;
            if (i >= 0 && i < n3) cgt[((size_t)j * n2 + k) * n3 + i] = clebsch(l1, j - l1, l2, k - l2, l3, i - l3);
        }
    std::vector<double> Q((size_t)n1 * n2 * n3, 0.0);
    const bool even = ((l1 + l2 + l3) & 1) == 0;
    for (int a = 0; a < n1; ++a)
        for (int b = 0; b < n2; ++b)
            for (int c = 0; c < n3; ++c) {
                std::complex<ld> s = 0.0L;
                for (int j = 0; j < n1; ++j) {
                    const std::complex<ld> u1 = std::conj(U1[(size_t)a * n1 + j]);
                    if (u1 == std::complex<ld>(0.0L)) continue;
                    for (int k = 0; k < n2; ++k) {
                        const int i = (j - l1) + (k - l2) + l3;
                        if (i < 0 || i >= n3) continue;
                        s += U3[(size_t)c * n3 + i] * u1 * std::conj(U2[(size_t)b * n2 + k]) *
                             cgt[((size_t)j * n2 + k) * n3 + i];
                    }
                }
                Q[((size_t)a * n2 + b) * n3 + c] = (double)(even ? s.real() : s.imag());
            }
    return cache.emplace(key, std::move(Q)).first->second;
}

struct Nz {
    int a, b, c;
    double v;
};

std::vector<Nz> nonzeros(int l1, int l2, int l3) {
    const auto& Q = coupling(l1, l2, l3);
    const int n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
    std::vector<Nz> out;
    for (size_t t = 0; t < Q.size(); ++t)
        if (std::fabs(Q[t]) > 1e-14) out.push_back({(int)(t / ((size_t)n2 * n3)), (int)(t / n3 % n2), (int)(t % n3), Q[t]});
    return out;
}

// ---------------------------------------------------------------------------
// Host: the tables of one (L, Lf)
// ---------------------------------------------------------------------------
// The node sums are kept in fp64: the terms of the expansion grow as
// |x - o|^lam |o - x_i|^mu while their sum is of order |r_ij|^l2, so fp32
// node sums would lose about (graph radius / neighbour distance)^Lf of
// their precision to cancellation (measured: 2.5e-3 relative at Lf = 8 on
// molecules of radius about 9 A).
struct NodeEntry {  // z[o] += c x[xi] S[si]
    int xi, si;
    double c;
};
struct OutEntry {  // out[u] += c w[p] Z[o] S[s]
    int o, sp;     // sp = s | p << 16
    double c;
};

struct Tables {
    int L = 0, Lf = 0, n_paths = 0, zdim = 0;
    std::vector<int> node_ptr;  // [zdim + 1]
    std::vector<NodeEntry> node;
    std::vector<int> out_ptr;   // [(L+1)^2 + 1]
    std::vector<OutEntry> out;
    bool ok = false;
};

int n_paths(int L, int Lf) {
    int n = 0;
    for (int l1 = 0; l1 <= L; ++l1)
        for (int l3 = 0; l3 <= L; ++l3)
            for (int l2 = std::abs(l1 - l3); l2 <= std::min(l1 + l3, Lf); ++l2) ++n;
    return n;
}

std::unique_ptr<Tables> build_tables(int L, int Lf) {
    auto T = std::make_unique<Tables>();
    T->L = L;
    T->Lf = Lf;
    struct Term {
        int p, l1, lam, k, mu, l3;
        double coef;
    };
    std::vector<Term> terms;
    std::map<std::tuple<int, int, int>, int> block;  // (l1, lam, k) -> z offset, filled below
    int p = 0;
    for (int l1 = 0; l1 <= L; ++l1)
        for (int l3 = 0; l3 <= L; ++l3)
            for (int l2 = std::abs(l1 - l3); l2 <= std::min(l1 + l3, Lf); ++l2, ++p) {
                const int n1 = 2 * l1 + 1, n3 = 2 * l3 + 1;
                const auto q123 = nonzeros(l1, l2, l3);
                for (int lam = 0; lam <= l2; ++lam) {
                    const int mu = l2 - lam, nl = 2 * lam + 1, nm = 2 * mu + 1;
                    // TA[m1][ml][mm][m3] = sum_m2 Q^{l1 l2 l3}[m1][m2][m3] Q^{lam mu l2}[ml][mm][m2]
                    std::vector<double> TA((size_t)n1 * nl * nm * n3, 0.0), rebuilt(TA.size(), 0.0);
                    const auto& Qlm = coupling(lam, mu, l2);
                    for (const Nz& e : q123)
                        for (int ml = 0; ml < nl; ++ml)
                            for (int mm = 0; mm < nm; ++mm) {
                                const double v = Qlm[((size_t)ml * nm + mm) * (2 * l2 + 1) + e.b];
                                if (v != 0.0) TA[(((size_t)e.a * nl + ml) * nm + mm) * n3 + e.c] += e.v * v;
                            }
                    const double kappa = std::sqrt((double)(fact(2 * l2) / (fact(2 * lam) * fact(2 * l2 - 2 * lam))));
                    for (int k = std::abs(l1 - lam); k <= l1 + lam; ++k) {
                        if (k < std::abs(mu - l3) || k > mu + l3) continue;
                        // TB_k[m1][ml][mm][m3] = sum_mk Q^{l1 lam k}[m1][ml][mk] Q^{k mu l3}[mk][mm][m3]
                        const auto q1 = nonzeros(l1, lam, k), q2 = nonzeros(k, mu, l3);
                        double ck = 0.0;
                        for (const Nz& a : q1)
                            for (const Nz& b : q2)
                                if (b.a == a.c) ck += a.v * b.v * TA[(((size_t)a.a * nl + a.b) * nm + b.b) * n3 + b.c];
                        ck /= (double)n3;
                        if (std::fabs(ck) < 1e-12) continue;
                        for (const Nz& a : q1)
                            for (const Nz& b : q2)
                                if (b.a == a.c) rebuilt[(((size_t)a.a * nl + a.b) * nm + b.b) * n3 + b.c] += ck * a.v * b.v;
                        block[std::make_tuple(l1, lam, k)] = 0;
                        terms.push_back({p, l1, lam, k, mu, l3, kappa * ck});
                    }
                    for (size_t t = 0; t < TA.size(); ++t)
                        if (std::fabs(TA[t] - rebuilt[t]) > 1e-9) return T;  // not ok: the schemes do not match
                }
            }
    T->n_paths = p;
    int off = 0;
    for (auto& kv : block) {
        kv.second = off;
        off += 2 * std::get<2>(kv.first) + 1;
    }
    T->zdim = off;
    // node table: z[(l1, lam, k), mk] = sum Q^{l1 lam k}[m1][ml][mk] x[l1, m1] S^lam[ml]
    T->node_ptr.assign(off + 1, 0);
    std::vector<std::vector<NodeEntry>> per(off);
    for (const auto& kv : block) {
        const int l1 = std::get<0>(kv.first), lam = std::get<1>(kv.first), k = std::get<2>(kv.first);
        for (const Nz& e : nonzeros(l1, lam, k))
            per[kv.second + e.c].push_back({l1 * l1 + e.a, lam * lam + e.b, e.v});
    }
    for (int o = 0; o < off; ++o) {
        T->node_ptr[o + 1] = T->node_ptr[o] + (int)per[o].size();
        T->node.insert(T->node.end(), per[o].begin(), per[o].end());
    }
    // output table: out[l3, m3] += coef Q^{k mu l3}[mk][mm][m3] w[p] Z[(l1, lam, k), mk] S^mu[mm]
    const int K = (L + 1) * (L + 1);
    std::vector<std::vector<OutEntry>> po(K);
    for (const Term& t : terms) {
        const int base = block.at(std::make_tuple(t.l1, t.lam, t.k));
        for (const Nz& e : nonzeros(t.k, t.mu, t.l3))
            po[t.l3 * t.l3 + e.c].push_back({base + e.a, (t.mu * t.mu + e.b) | (t.p << 16), t.coef * e.v});
    }
    T->out_ptr.assign(K + 1, 0);
    for (int u = 0; u < K; ++u) {
        T->out_ptr[u + 1] = T->out_ptr[u] + (int)po[u].size();
        T->out.insert(T->out.end(), po[u].begin(), po[u].end());
    }
    T->ok = true;
    return T;
}

const Tables* tables(int L, int Lf) {
    static std::mutex mu;
    static std::map<std::pair<int, int>, std::unique_ptr<Tables>> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(L, Lf);
    auto it = cache.find(key);
    if (it == cache.end()) it = cache.emplace(key, build_tables(L, Lf)).first;
    return it->second->ok ? it->second.get() : nullptr;
}

// ---------------------------------------------------------------------------
// Host and device: solid harmonics, radial basis, logits
// ---------------------------------------------------------------------------

// S^l_m(x, y, z), l <= lmax, flat index l*l + l + m: S^l_0 = T_l^0,
// S^l_{+-m} = sqrt(2 (l-m)!/(l+m)!) T_l^m {Re, Im}(x + i y)^m, where
// T_l^m = r^(l-m) P_l^(m)(z/r) (the m-th derivative of the Legendre
// polynomial) follows T_m^m = (2m-1)!!, T_{m+1}^m = (2m+1) z T_m^m,
// (l-m) T_l^m = (2l-1) z T_{l-1}^m - (l+m-1) r^2 T_{l-2}^m.
__host__ __device__ inline void solid_harmonics(int lmax, double x, double y, double z, double* S) {
    const double r2 = x * x + y * y + z * z;
    double cm = 1.0, sm = 0.0, dfact = 1.0;
    for (int m = 0; m <= lmax; ++m) {
        double t1 = 0.0, t2 = 0.0;  // T_{l-1}^m, T_{l-2}^m
        for (int l = m; l <= lmax; ++l) {
            double t;
            if (l == m)
                t = dfact;
            else if (l == m + 1)
                t = (double)(2 * m + 1) * z * t1;
            else
                t = ((double)(2 * l - 1) * z * t1 - (double)(l + m - 1) * r2 * t2) / (double)(l - m);
            t2 = t1;
            t1 = t;
            if (m == 0) {
                S[l * l + l] = t;
            } else {
                double f = 1.0;
                for (int q = l - m + 1; q <= l + m; ++q) f *= (double)q;
                const double nrm = sqrt(2.0 / f);
                S[l * l + l + m] = nrm * t * cm;
                S[l * l + l - m] = nrm * t * sm;
            }
        }
        const double c2 = x * cm - y * sm, s2 = x * sm + y * cm;
        cm = c2;
        sm = s2;
        dfact *= (double)(2 * m + 1);
    }
}

struct Params {
    int N, L, Lf, C, H, n_rbf, zdim, K;
    float cutoff;
    const float* pos;
    const int32_t* graph_ptr;
    int n_graphs;
    const int32_t* row_ptr;
    const int32_t* col;
    const float* x;
    const float* Wq;
    const float* Wk;
    const float* Wrad;
    const float* w;
    float* out;
    const int* node_ptr;
    const NodeEntry* node;
    const int* out_ptr;
    const OutEntry* outt;
    double* rel;
    float* q;
    float* k;
    double* z;
    double* Z;
};

// a_ij^h = g_a^h(d) <q_i^h, k_j^h> / sqrt(C/H), g_a = rho(d) W_rad,
// rho_k(d) = u(d) exp(-((d - k rc/(n-1)) / (rc/(n-1)))^2), u = (cos(pi d/rc) + 1)/2
__host__ __device__ inline float logit(const Params& P, int i, int j, int h) {
    const float dx = P.pos[3 * j] - P.pos[3 * i], dy = P.pos[3 * j + 1] - P.pos[3 * i + 1],
                dz = P.pos[3 * j + 2] - P.pos[3 * i + 2];
    const float d = sqrtf(dx * dx + dy * dy + dz * dz);
    const float step = P.cutoff / (float)(P.n_rbf - 1);
    const float u = 0.5f * (cosf(3.14159265358979323846f * d / P.cutoff) + 1.f);
    float ga = 0.f;
    for (int kb = 0; kb < P.n_rbf; ++kb) {
        const float t = (d - (float)kb * step) / step;
        ga += u * expf(-t * t) * P.Wrad[kb * P.H + h];
    }
    const int dh = P.C / P.H;
    const float* qi = P.q + (size_t)i * P.C + h * dh;
    const float* kj = P.k + (size_t)j * P.C + h * dh;
    float dot = 0.f;
    for (int c = 0; c < dh; ++c) dot += qi[c] * kj[c];
    return ga * dot / sqrtf((float)dh);
}

// z_j[o][c] for one channel, given S = S(a_j)
__host__ __device__ inline void node_products(const Params& P, int j, int c, const double* S) {
    const float* xj = P.x + (size_t)j * P.K * P.C + c;
    double* zj = P.z + (size_t)j * P.zdim * P.C + c;
    for (int o = 0; o < P.zdim; ++o) {
        double acc = 0.0;
        for (int e = P.node_ptr[o]; e < P.node_ptr[o + 1]; ++e) {
            const NodeEntry t = P.node[e];
            acc += t.c * (double)xj[(size_t)t.xi * P.C] * S[t.si];
        }
        zj[(size_t)o * P.C] = acc;
    }
}

// out_i[u][c] for one channel, given S = S(b_i)
__host__ __device__ inline void out_products(const Params& P, int i, int c, const double* S) {
    const double* Zi = P.Z + (size_t)i * P.zdim * P.C + c;
    float* oi = P.out + (size_t)i * P.K * P.C + c;
    for (int u = 0; u < P.K; ++u) {
        double acc = 0.0;
        for (int e = P.out_ptr[u]; e < P.out_ptr[u + 1]; ++e) {
            const OutEntry t = P.outt[e];
            acc += t.c * (double)P.w[(size_t)(t.sp >> 16) * P.C + c] * Zi[(size_t)t.o * P.C] * S[t.sp & 0xffff];
        }
        oi[(size_t)u * P.C] = (float)acc;
    }
}

// ---------------------------------------------------------------------------
// Kernels
// ---------------------------------------------------------------------------

// rel = x - o for the atoms of graph blockIdx.x, o the graph's mean position
__global__ void k_sixj_rel(Params P) {
    const int g = blockIdx.x;
    // a graph range outside [0, N] is clamped into it (no access outside pos and rel)
    const int b = P.graph_ptr ? min(max(P.graph_ptr[g], 0), P.N) : 0;
    const int e = P.graph_ptr ? min(max(P.graph_ptr[g + 1], b), P.N) : P.N;
    __shared__ double red[3][256];
    double s[3] = {0.0, 0.0, 0.0};
    for (int n = b + threadIdx.x; n < e; n += blockDim.x)
        for (int a = 0; a < 3; ++a) s[a] += (double)P.pos[3 * n + a];
    for (int a = 0; a < 3; ++a) red[a][threadIdx.x] = s[a];
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w)
            for (int a = 0; a < 3; ++a) red[a][threadIdx.x] += red[a][threadIdx.x + w];
        __syncthreads();
    }
    const int cnt = e - b;
    for (int n = b + threadIdx.x; n < e; n += blockDim.x)
        for (int a = 0; a < 3; ++a) P.rel[3 * n + a] = (double)P.pos[3 * n + a] - red[a][0] / (double)cnt;
}

// q = W_q x[l=0], k = W_k x[l=0]
__global__ void k_sixj_qk(Params P) {
    const int i = blockIdx.x;
    for (int c = threadIdx.x; c < 2 * P.C; c += blockDim.x) {
        const int cc = c % P.C;
        const float* W = (c < P.C ? P.Wq : P.Wk) + (size_t)cc * P.C;
        const float* x0 = P.x + (size_t)i * P.K * P.C;
        float s = 0.f;
        for (int t = 0; t < P.C; ++t) s += W[t] * x0[t];
        (c < P.C ? P.q : P.k)[(size_t)i * P.C + cc] = s;
    }
}

__global__ void k_sixj_node(Params P) {
    __shared__ double S[(kMaxLf + 1) * (kMaxLf + 1)];
    const int j = blockIdx.x;
    if (threadIdx.x == 0) solid_harmonics(P.Lf, P.rel[3 * j], P.rel[3 * j + 1], P.rel[3 * j + 2], S);
    __syncthreads();
    for (int c = threadIdx.x; c < P.C; c += blockDim.x) node_products(P, j, c, S);
}

// Z_i = sum_j softmax_j(a_ij^{h(c)}) z_j: two passes over the edges (max and
// sum per head), then the weighted sum in chunks of kAggE edges; each thread
// owns the same elements of Z_i in every chunk
__global__ void __launch_bounds__(256) k_sixj_agg(Params P) {
    __shared__ float red[2][256];
    __shared__ float lse[kMaxH];
    __shared__ float al[kAggE][kMaxH];
    __shared__ int jn[kAggE];
    const int i = blockIdx.x, tid = threadIdx.x, nt = blockDim.x, H = P.H, dh = P.C / P.H;
    const int e0 = P.row_ptr[i], deg = P.row_ptr[i + 1] - e0;
    const size_t zsz = (size_t)P.zdim * P.C;
    double* Zi = P.Z + (size_t)i * zsz;
    if (deg == 0) {
        for (size_t t = tid; t < zsz; t += nt) Zi[t] = 0.0;
        return;
    }
    {
        // thread t: head t % H, edges t / H, t / H + nt / H, ...
        const int h = tid % H;
        float mh = -INFINITY, sh = 0.f;
        if (tid < (nt / H) * H)
            for (int e = tid / H; e < deg; e += nt / H) {
                const float a = logit(P, i, P.col[e0 + e], h);
                const float mn = fmaxf(mh, a);
                sh = sh * expf(mh - mn) + expf(a - mn);
                mh = mn;
            }
        red[0][tid] = mh;
        red[1][tid] = sh;
    }
    __syncthreads();
    if (tid < H) {
        float mh = -INFINITY, sh = 0.f;
        for (int t = tid; t < (nt / H) * H; t += H) {
            const float mo = red[0][t], so = red[1][t];
            if (mo == -INFINITY) continue;
            const float mn = fmaxf(mh, mo);
            sh = (mh == -INFINITY ? 0.f : sh * expf(mh - mn)) + so * expf(mo - mn);
            mh = mn;
        }
        lse[tid] = mh + logf(sh);
    }
    __syncthreads();
    for (int c0 = 0; c0 < deg; c0 += kAggE) {
        const int ne = min(kAggE, deg - c0);
        for (int t = tid; t < ne * H; t += nt) {
            const int e = t / H, h = t % H;
            const int j = P.col[e0 + c0 + e];
            al[e][h] = expf(logit(P, i, j, h) - lse[h]);
            if (h == 0) jn[e] = j;
        }
        __syncthreads();
        for (size_t t = tid; t < zsz; t += nt) {
            const int h = (int)(t % P.C) / dh;
            double acc = c0 == 0 ? 0.0 : Zi[t];
            for (int e = 0; e < ne; ++e) acc += (double)al[e][h] * P.z[(size_t)jn[e] * zsz + t];
            Zi[t] = acc;
        }
        __syncthreads();
    }
}

__global__ void k_sixj_out(Params P) {
    __shared__ double S[(kMaxLf + 1) * (kMaxLf + 1)];
    const int i = blockIdx.x;
    if (threadIdx.x == 0) solid_harmonics(P.Lf, -P.rel[3 * i], -P.rel[3 * i + 1], -P.rel[3 * i + 2], S);
    __syncthreads();
    for (int c = threadIdx.x; c < P.C; c += blockDim.x) out_products(P, i, c, S);
}

struct Layout {
    size_t node_ptr, node, out_ptr, outt, rel, q, k, z, Z, bytes;
};

Layout layout(int64_t N, const e2f_sixj_cfg& c, const Tables& T) {
    Layout w{};
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off = align_up(off + b, 256);
        return o;
    };
    const int K = (c.L + 1) * (c.L + 1);
    w.node_ptr = take(sizeof(int) * T.node_ptr.size());
    w.node = take(sizeof(NodeEntry) * std::max<size_t>(T.node.size(), 1));
    w.out_ptr = take(sizeof(int) * (size_t)(K + 1));
    w.outt = take(sizeof(OutEntry) * std::max<size_t>(T.out.size(), 1));
    w.rel = take(sizeof(double) * 3 * (size_t)N);
    w.q = take(sizeof(float) * (size_t)N * c.C);
    w.k = take(sizeof(float) * (size_t)N * c.C);
    w.z = take(sizeof(double) * (size_t)N * T.zdim * c.C);
    w.Z = take(sizeof(double) * (size_t)N * T.zdim * c.C);
    w.bytes = off;
    return w;
}

bool shape_ok(const e2f_sixj_cfg& c) {
    return c.L >= 0 && c.L <= kMaxL && c.Lf >= 0 && c.Lf <= 2 * c.L && c.C >= 1 && c.C <= 256 && c.H >= 1 &&
           c.H <= kMaxH && c.C % c.H == 0 && c.n_rbf >= 2 && c.n_rbf <= kMaxRbf && c.cutoff > 0.f;
}

}  // namespace sixj
}  // namespace e2f

using namespace e2f;
using namespace e2f::sixj;

extern "C" int e2f_sixj_n_paths(int L, int Lf) {
    if (L < 0 || L > kMaxL || Lf < 0 || Lf > 2 * L) return -1;
    return n_paths(L, Lf);
}

extern "C" size_t e2f_sixj_workspace_size(int64_t n_atoms, const e2f_sixj_cfg* cfg) {
    if (!cfg || n_atoms < 0 || !shape_ok(*cfg)) return 0;
    const Tables* T = tables(cfg->L, cfg->Lf);
    if (!T) return 0;
    return layout(n_atoms, *cfg, *T).bytes;
}

extern "C" e2f_status e2f_sixj_attention(const e2f_sixj_cfg* cfg, const float* pos, int64_t n_atoms,
                                         const int32_t* graph_ptr, int32_t n_graphs, const int32_t* row_ptr,
                                         const int32_t* col, int64_t n_pairs, const float* x, const float* W_q,
                                         const float* W_k, const float* W_rad, const float* w_path, float* out,
                                         void* workspace, size_t ws_bytes, void* stream) {
    if (!cfg || n_atoms < 0 || n_pairs < 0) return E2F_ERR_INVALID_ARG;
    if (!shape_ok(*cfg)) return E2F_ERR_UNSUPPORTED;
    if (n_atoms > INT32_MAX || n_pairs > INT32_MAX) return E2F_ERR_UNSUPPORTED;
    if (graph_ptr && n_graphs < 1) return E2F_ERR_INVALID_ARG;
    if (n_atoms == 0) return E2F_OK;
    if (!pos || !row_ptr || (n_pairs > 0 && !col) || !x || !W_q || !W_k || !W_rad || !w_path || !out || !workspace)
        return E2F_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return E2F_ERR_ALIGNMENT;
    const Tables* T = tables(cfg->L, cfg->Lf);
    if (!T) return E2F_ERR_UNSUPPORTED;
    const Layout Lw = layout(n_atoms, *cfg, *T);
    if (ws_bytes < Lw.bytes) return E2F_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    Params P{};
    P.N = (int)n_atoms;
    P.L = cfg->L;
    P.Lf = cfg->Lf;
    P.C = cfg->C;
    P.H = cfg->H;
    P.n_rbf = cfg->n_rbf;
    P.zdim = T->zdim;
    P.K = (cfg->L + 1) * (cfg->L + 1);
    P.cutoff = cfg->cutoff;
    P.pos = pos;
    P.graph_ptr = graph_ptr;
    P.n_graphs = graph_ptr ? n_graphs : 1;
    P.row_ptr = row_ptr;
    P.col = col;
    P.x = x;
    P.Wq = W_q;
    P.Wk = W_k;
    P.Wrad = W_rad;
    P.w = w_path;
    P.out = out;
    P.node_ptr = reinterpret_cast<const int*>(ws + Lw.node_ptr);
    P.node = reinterpret_cast<const NodeEntry*>(ws + Lw.node);
    P.out_ptr = reinterpret_cast<const int*>(ws + Lw.out_ptr);
    P.outt = reinterpret_cast<const OutEntry*>(ws + Lw.outt);
    P.rel = reinterpret_cast<double*>(ws + Lw.rel);
    P.q = reinterpret_cast<float*>(ws + Lw.q);
    P.k = reinterpret_cast<float*>(ws + Lw.k);
    P.z = reinterpret_cast<double*>(ws + Lw.z);
    P.Z = reinterpret_cast<double*>(ws + Lw.Z);
    // the tables live in the process-wide cache for the rest of the process,
    // so the copies may stay in flight after this call returns
    E2F_CUDA_TRY(cudaMemcpyAsync(ws + Lw.node_ptr, T->node_ptr.data(), sizeof(int) * T->node_ptr.size(),
                                 cudaMemcpyHostToDevice, s));
    if (!T->node.empty())
        E2F_CUDA_TRY(cudaMemcpyAsync(ws + Lw.node, T->node.data(), sizeof(NodeEntry) * T->node.size(),
                                     cudaMemcpyHostToDevice, s));
    E2F_CUDA_TRY(cudaMemcpyAsync(ws + Lw.out_ptr, T->out_ptr.data(), sizeof(int) * T->out_ptr.size(),
                                 cudaMemcpyHostToDevice, s));
    if (!T->out.empty())
        E2F_CUDA_TRY(cudaMemcpyAsync(ws + Lw.outt, T->out.data(), sizeof(OutEntry) * T->out.size(),
                                     cudaMemcpyHostToDevice, s));
    const int nt = std::min(256, (P.C + 31) / 32 * 32);
    count_launch();
    k_sixj_rel<<<P.n_graphs, 256, 0, s>>>(P);
    count_launch();
    k_sixj_qk<<<P.N, 256, 0, s>>>(P);
    count_launch();
    k_sixj_node<<<P.N, nt, 0, s>>>(P);
    count_launch();
    k_sixj_agg<<<P.N, 256, 0, s>>>(P);
    count_launch();
    k_sixj_out<<<P.N, nt, 0, s>>>(P);
    E2F_CUDA_TRY(cudaGetLastError());
    return E2F_OK;
}
