// encode.cpp -- the CPU packer ep_encode_tensor (threaded C++17).
//
// EntroPack paper §3.1 pipeline: row normalisation, sampled-row scale search
// (§3.4 "Geometric search", App. C.1), full-tensor E8 quantisation (§1, Conway &
// Sloane 1982), row-scale refit (§3.5), seventeen coset-conditioned frequency
// tables (§3.6, App. A.3) and tiled interleaved rANS (§3.6, App. C.3).
//
// The readings of the pages that the decoder does not see (row normaliser, tie
// rules, table normalisation, sample generator) are fixed so that the same input
// gives the same bytes on every run and every thread count.  Rows, samples and
// tiles are spread over threads; every floating-point sum is taken in index order
// inside one row, so threading never changes a result.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <new>
#include <queue>
#include <thread>
#include <vector>

#include "entropack.h"
#include "ep_format.h"
#include "encode_host.h"

namespace ep {
namespace {

using host::Hist;
using host::normalise;
using host::rdo_ratios;
using host::Table;
using host::tile_symbols_for;

// ------------------------------------------------------------------ threads

void parallel_for(int64_t n, int nthreads, const std::function<void(int64_t, int64_t)>& fn) {
    if (n <= 0) return;
    int nt = (int)std::min<int64_t>(nthreads, n);
    if (nt <= 1) {
        fn(0, n);
        return;
    }
    // dynamic chunks keep threads busy when rows or tiles differ in cost
    const int64_t chunk = std::max<int64_t>(1, n / (int64_t)(nt * 8));
    std::atomic<int64_t> next(0);
    std::vector<std::thread> th;
    th.reserve(nt);
    for (int i = 0; i < nt; ++i)
        th.emplace_back([&]() {
            for (;;) {
                const int64_t a = next.fetch_add(chunk);
                if (a >= n) break;
                fn(a, std::min(n, a + chunk));
            }
        });
    for (auto& t : th) t.join();
}

// ------------------------------------------------------------ the quantiser

// Nearest point of D8 (integer vectors, even sum): round to nearest (ties to
// even); if the sum is odd, move the coordinate furthest from its rounding one
// step the other way (first such coordinate; up when u - a >= 0).
inline void d8_nearest(const double* u, double* a) {
    long long par = 0;
    int far_k = 0;
    double far_d = -1.0;
    for (int k = 0; k < 8; ++k) {
        a[k] = std::nearbyint(u[k]);
        par += (long long)a[k];
        const double d = std::fabs(u[k] - a[k]);
        if (d > far_d) {
            far_d = d;
            far_k = k;
        }
    }
    if (par & 1LL) a[far_k] += (u[far_k] - a[far_k] >= 0.0) ? 1.0 : -1.0;
}

// E8 = D8 u (D8 + 1/2): the nearer coset decoding; ties to D8.  Writes the
// field tuple (c, z1..z7, m) of the chosen point and its coordinates y.
inline void e8_fields(const double* u, int32_t* f, double* y) {
    double a[8], h[8], v[8];
    d8_nearest(u, a);
    for (int k = 0; k < 8; ++k) v[k] = u[k] - 0.5;
    d8_nearest(v, h);
    double da = 0.0, dh = 0.0;
    for (int k = 0; k < 8; ++k) {
        const double ea = u[k] - a[k];
        const double eh = u[k] - (h[k] + 0.5);
        da += ea * ea;
        dh += eh * eh;
    }
    const int c = dh < da ? 1 : 0;
    const double* z = c ? h : a;  // z = y - c/2 is the D8 point in both cosets
    long long s7 = 0;
    for (int k = 0; k < 7; ++k) {
        f[1 + k] = (int32_t)z[k];
        s7 += (long long)z[k];
    }
    const long long z8 = (long long)z[7];
    f[0] = c;
    f[8] = (int32_t)((z8 - (s7 & 1LL)) / 2);  // parity reduction: m = (z8 - p) / 2
    for (int k = 0; k < 8; ++k) y[k] = z[k] + 0.5 * c;
}

// Quantise one row at scale s: u = (w / n) / s, a partial last vector padded
// with zeros; fields into f (9 per vector); optional refit sums <w, y> and
// <y, y> over the real entries in index order.
void quantize_row(const float* w, int64_t cols, double n, double s, int32_t* f, double* num, double* den) {
    double u[8], y[8];
    double sn = 0.0, sd = 0.0;
    for (int64_t q = 0; q < (cols + 7) / 8; ++q) {
        const int real = (int)std::min<int64_t>(8, cols - 8 * q);
        for (int k = 0; k < 8; ++k) u[k] = k < real ? ((double)w[8 * q + k] / n) / s : 0.0;
        e8_fields(u, f + kFields * q, y);
        if (num) {
            for (int k = 0; k < real; ++k) {
                sn += (double)w[8 * q + k] * y[k];
                sd += y[k] * y[k];
            }
        }
    }
    if (num) {
        *num = sn;
        *den = sd;
    }
}

// --------------------------------------------------------------- the model

// alphabets ([min, max] per table) of vectors [0, nvec): contiguous parts per thread, then merged
Hist alphabet_of(const int32_t* f, int64_t nvec, int nthreads) {
    const int nt = std::max(1, (int)std::min<int64_t>(nthreads, (nvec + 65535) / 65536));
    std::vector<Hist> part(nt);
    const int64_t per = (nvec + nt - 1) / nt;
    std::vector<std::thread> th;
    for (int i = 0; i < nt; ++i)
        th.emplace_back([&, i]() {
            part[i].reset();
            const int64_t a = i * per, e = std::min(nvec, a + per);
            if (e > a) part[i].add_range(f + kFields * a, e - a);
        });
    for (auto& t : th) t.join();
    Hist all;
    all.reset();
    for (auto& h : part) all.merge(h);
    return all;
}

// counts of the fields of vectors [0, nvec) into tables with the given alphabets
void count_fields(const int32_t* f, int64_t nvec, const Hist& al, Table* tabs, int nthreads) {
    for (int t = 0; t < kTables; ++t) {
        tabs[t].A = (uint32_t)al.alpha(t);
        tabs[t].min = tabs[t].A ? (int32_t)al.lo[t] : 0;
        tabs[t].total = 0;
        tabs[t].count.assign(std::max<uint32_t>(tabs[t].A, 1), 0);
    }
    const int nt = std::max(1, (int)std::min<int64_t>(nthreads, (nvec + 65535) / 65536));
    std::vector<std::vector<uint64_t>> part(nt);
    size_t tot = 0;
    std::vector<size_t> base(kTables + 1, 0);
    for (int t = 0; t < kTables; ++t) {
        base[t] = tot;
        tot += tabs[t].count.size();
    }
    base[kTables] = tot;
    const int64_t per = (nvec + nt - 1) / nt;
    std::vector<std::thread> th;
    for (int i = 0; i < nt; ++i) {
        th.emplace_back([&, i]() {
            std::vector<uint64_t>& c = part[i];
            c.assign(tot, 0);
            const int64_t a = i * per, b = std::min(nvec, a + per);
            for (int64_t g = a; g < b; ++g) {
                const int32_t* v = f + kFields * g;
                for (int k = 0; k < kFields; ++k) {
                    const int t = table_index(k, v[0]);
                    c[base[t] + (size_t)(v[k] - tabs[t].min)] += 1;
                }
            }
        });
    }
    for (auto& t : th) t.join();
    for (int t = 0; t < kTables; ++t)
        for (size_t s = 0; s < tabs[t].count.size(); ++s) {
            uint64_t v = 0;
            for (int i = 0; i < nt; ++i) v += part[i][base[t] + s];
            tabs[t].count[s] = v;
            tabs[t].total += v;
        }
}

// ------------------------------------------------- per-row refinement (RDO)

// Ideal code length of one row's fields under the tables, symbols in order; a
// symbol the tables give no frequency costs b bits.
double row_bits(const int32_t* f, int64_t nq, const Table* tabs, int b) {
    double bits = 0.0;
    for (int64_t q = 0; q < nq; ++q) {
        const int32_t* v = f + kFields * q;
        for (int k = 0; k < kFields; ++k) {
            const Table& tb = tabs[table_index(k, v[0])];
            const int64_t i = (int64_t)v[k] - tb.min;
            const uint32_t fr = (tb.A && i >= 0 && i < (int64_t)tb.A) ? tb.freq[(size_t)i] : 0u;
            bits += (double)b - std::log2((double)(fr ? fr : 1u));
        }
    }
    return bits;
}

// Tables (alphabets, counts, frequencies at 2^b) of the given fields.
void build_tables(const int32_t* f, int64_t nvec, int b, int nthreads, Table* tabs) {
    const Hist al = alphabet_of(f, nvec, nthreads);
    count_fields(f, nvec, al, tabs, nthreads);
    for (int t = 0; t < kTables; ++t) normalise(tabs[t], b);
}

// App. C.2 allocation: every candidate of every row quantised at rho_k s and
// refitted, its distortion sum (w - sigma y)^2; admissible when its symbols lie
// in the baseline alphabets.  A sweep prices the candidates under the current
// tables, bisects log2 lambda on [-80, 80] (64 steps) for the smallest lambda
// whose choices argmin D + lambda R (ties: lowest k) fit the baseline's ideal
// code length, and rebuilds the tables from the choices.  `fields` holds the
// ratio-1 fields on entry and the chosen ones on return; `scales` the chosen
// row scales.  Sums run in the same order as the documented algorithm.
void rdo_refine(const float* W, int64_t rows, int64_t cols, const std::vector<double>& norms, double s, int b, int K,
                int sweeps, int nthreads, std::vector<int32_t>& fields, std::vector<float>& scales) {
    const int64_t nq = (cols + 7) / 8, nvec = rows * nq, rowf = kFields * nq;
    if (K > 64) K = 64;
    double rho[64];
    rdo_ratios(K, rho);
    std::vector<int32_t> cf((size_t)(K * rows * rowf));
    std::vector<float> cs((size_t)(K * rows));
    std::vector<double> cd((size_t)(K * rows)), cr((size_t)(K * rows)), rsel((size_t)rows);
    std::vector<uint8_t> ok((size_t)(K * rows));
    std::vector<int> sel((size_t)rows, 0);
    Table base[kTables];
    build_tables(fields.data(), nvec, b, nthreads, base);
    parallel_for(rows, nthreads, [&](int64_t a, int64_t e) {
        std::vector<double> y((size_t)(8 * nq));
        double u[8];
        for (int64_t r = a; r < e; ++r) {
            const float* w = W + r * cols;
            for (int k = 0; k < K; ++k) {
                const double sk = rho[k] * s;
                int32_t* f = cf.data() + (size_t)((k * rows + r) * rowf);
                double num = 0.0, den = 0.0;
                for (int64_t q = 0; q < nq; ++q) {
                    for (int i = 0; i < 8; ++i) u[i] = 8 * q + i < cols ? ((double)w[8 * q + i] / norms[r]) / sk : 0.0;
                    e8_fields(u, f + kFields * q, y.data() + 8 * q);
                }
                for (int64_t j = 0; j < cols; ++j) {
                    num += (double)w[j] * y[j];
                    den += y[j] * y[j];
                }
                const float sg = den == 0.0 ? 0.0f : (float)(num / den);
                double d = 0.0;
                for (int64_t j = 0; j < cols; ++j) {
                    const double er = (double)w[j] - (double)sg * y[j];
                    d += er * er;
                }
                uint8_t in = 1;
                for (int64_t q = 0; q < nq && in; ++q)
                    for (int m = 0; m < kFields; ++m) {
                        const Table& tb = base[table_index(m, f[kFields * q])];
                        const int64_t i = (int64_t)f[kFields * q + m] - tb.min;
                        if (!tb.A || i < 0 || i >= (int64_t)tb.A) in = 0;
                    }
                cs[(size_t)(k * rows + r)] = sg;
                cd[(size_t)(k * rows + r)] = d;
                ok[(size_t)(k * rows + r)] = in;
            }
        }
    });
    parallel_for(rows, nthreads, [&](int64_t a, int64_t e) {
        for (int64_t r = a; r < e; ++r) rsel[(size_t)r] = row_bits(cf.data() + (size_t)(r * rowf), nq, base, b);
    });
    double budget = 0.0;
    for (int64_t r = 0; r < rows; ++r) budget += rsel[(size_t)r];
    Table next[kTables];
    const Table* model = base;
    for (int sw = 0; sw < sweeps; ++sw) {
        parallel_for(rows, nthreads, [&](int64_t a, int64_t e) {
            for (int64_t r = a; r < e; ++r)
                for (int k = 0; k < K; ++k) {
                    const size_t i = (size_t)(k * rows + r);
                    cr[i] = ok[i] ? row_bits(cf.data() + (size_t)((k * rows + r) * rowf), nq, model, b) : INFINITY;
                }
        });
        host::rdo_bisect(cd.data(), cr.data(), rows, K, budget, nthreads, sel.data());
        parallel_for(rows, nthreads, [&](int64_t a, int64_t e) {
            for (int64_t r = a; r < e; ++r)
                std::memcpy(fields.data() + (size_t)(r * rowf), cf.data() + (size_t)((sel[(size_t)r] * rows + r) * rowf),
                            sizeof(int32_t) * (size_t)rowf);
        });
        build_tables(fields.data(), nvec, b, nthreads, next);
        model = next;
    }
    for (int64_t r = 0; r < rows; ++r) scales[(size_t)r] = cs[(size_t)(sel[(size_t)r] * rows + r)];
}

// ------------------------------------------------------------------- rANS

// Encode one tile (vectors [v0, v0 + vt)): steps in reverse, lanes in reverse
// inside a step, so that the decoder reads forward and in ascending lane order.
void encode_tile(const int32_t* fields, int64_t v0, int64_t vt, const Table* tabs, int b, std::vector<uint16_t>& out,
                 uint32_t* states) {
    const uint32_t M = 1u << b;
    uint64_t x[kLanes];
    for (int j = 0; j < kLanes; ++j) x[j] = kStateLow;
    const int64_t rounds = (vt + kLanes - 1) / kLanes;
    std::vector<uint16_t> rev;
    rev.reserve((size_t)(vt * 4));
    for (int64_t st = kFields * rounds - 1; st >= 0; --st) {
        const int64_t r = st / kFields;
        const int k = (int)(st % kFields);
        for (int j = kLanes - 1; j >= 0; --j) {
            const int64_t v = kLanes * r + j;
            if (v >= vt) continue;
            const int32_t* f = fields + kFields * (v0 + v);
            const Table& tb = tabs[table_index(k, f[0])];
            const uint32_t s = (uint32_t)(f[k] - tb.min);
            const uint64_t fr = tb.freq[s], cm = tb.cum[s];
            if (x[j] >= (fr << (31 - b))) {
                rev.push_back((uint16_t)(x[j] & 0xFFFFu));
                x[j] >>= 16;
            }
            x[j] = (x[j] / fr) * M + (x[j] % fr) + cm;
        }
    }
    out.assign(rev.rbegin(), rev.rend());
    for (int j = 0; j < kLanes; ++j) states[j] = (uint32_t)x[j];
}

// ---------------------------------------------------------------- the blob

struct Encoder {
    const float* W;
    int64_t rows, cols, nq, nvec;
    double target;
    int nthreads;
    bool container;
    int64_t ntiles;
    std::vector<double> norms;

    // Stored-size estimate from the sampled rows at (s, b); +inf when an alphabet exceeds 2^b.
    double estimate(const std::vector<int64_t>& srows, double s, int b, std::vector<int32_t>& sf) const {
        const int64_t rs = (int64_t)srows.size();
        parallel_for(rs, nthreads, [&](int64_t a, int64_t e) {
            for (int64_t i = a; i < e; ++i)
                quantize_row(W + srows[i] * cols, cols, norms[srows[i]], s, sf.data() + (size_t)(kFields * nq * i),
                             nullptr, nullptr);
        });
        const int64_t ns = rs * nq;
        const Hist al = alphabet_of(sf.data(), ns, nthreads);
        if (al.amax_coord() > (1ull << b)) return INFINITY;
        Table tabs[kTables];
        count_fields(sf.data(), ns, al, tabs, nthreads);
        return host::estimate_bpp(tabs, al, b, nvec, ns, ntiles, rows, cols, container);
    }
};

}  // namespace

// ------------------------------------------------ shared with the GPU encoder

namespace host {

// Paper §3.5, App. C.2: K candidate ratios in [0.70, 1.45]: 1 first, then the
// log-midpoint of the widest interval between neighbours and the range ends
// (ties: the lower interval); nested in K.
void rdo_ratios(int K, double* rho) {
    double pts[2 + 64];
    int n = 3;
    pts[0] = 0.70;
    pts[1] = 1.0;
    pts[2] = 1.45;
    rho[0] = 1.0;
    for (int k = 1; k < K && k < 64; ++k) {
        int best = 0;
        double wbest = -1.0;
        for (int i = 0; i + 1 < n; ++i) {
            const double w = std::log(pts[i + 1] / pts[i]);
            if (w > wbest) {
                wbest = w;
                best = i;
            }
        }
        const double mid = std::sqrt(pts[best] * pts[best + 1]);
        for (int i = n; i > best + 1; --i) pts[i] = pts[i - 1];
        pts[best + 1] = mid;
        ++n;
        rho[k] = mid;
    }
}

// Frequencies at M = 2^b: f = max(1, floor(count*M/total + 1/2)) for present
// symbols; the excess comes off the largest f > 1 one unit at a time (lowest
// symbol on ties), a shortfall goes to the most frequent symbol (lowest on ties).
void normalise(Table& tb, int b) {
    const uint32_t M = 1u << b;
    tb.freq.assign(std::max<uint32_t>(tb.A, 1), 0);
    tb.cum.assign(std::max<uint32_t>(tb.A, 1) + 1, 0);
    if (tb.A == 0) return;
    uint64_t sum = 0;
    for (uint32_t s = 0; s < tb.A; ++s) {
        if (tb.count[s]) {
            const double q = (double)tb.count[s] * (double)M / (double)tb.total;
            const double r = std::floor(q + 0.5);
            tb.freq[s] = r < 1.0 ? 1u : (uint32_t)r;
        }
        sum += tb.freq[s];
    }
    if (sum > M) {
        // max-heap on (f, -s): the same choice as a scan for the largest f > 1, lowest s
        auto cmp = [&](uint32_t x, uint32_t y) {
            return tb.freq[x] != tb.freq[y] ? tb.freq[x] < tb.freq[y] : x > y;
        };
        std::priority_queue<uint32_t, std::vector<uint32_t>, decltype(cmp)> pq(cmp);
        for (uint32_t s = 0; s < tb.A; ++s)
            if (tb.freq[s] > 1) pq.push(s);
        while (sum > M && !pq.empty()) {
            const uint32_t s = pq.top();
            pq.pop();
            tb.freq[s] -= 1;
            sum -= 1;
            if (tb.freq[s] > 1) pq.push(s);
        }
    }
    if (sum < M) {
        uint32_t best = 0;
        for (uint32_t s = 1; s < tb.A; ++s)
            if (tb.count[s] > tb.count[best]) best = s;
        tb.freq[best] += (uint32_t)(M - sum);
    }
    for (uint32_t s = 0; s < tb.A; ++s) tb.cum[s + 1] = tb.cum[s] + tb.freq[s];
}

void rdo_bisect(const double* cd, const double* cr, int64_t rows, int K, double budget, int nthreads, int* sel) {
    std::vector<double> rsel((size_t)rows);
    double lo = -80.0, hi = 80.0;
    for (int it = 0; it <= 64; ++it) {
        const double t = it < 64 ? 0.5 * (lo + hi) : hi;
        const double lam = std::exp2(t);
        parallel_for(rows, nthreads, [&](int64_t a, int64_t e) {
            for (int64_t r = a; r < e; ++r) {
                int best = 0;
                double jbest = cd[(size_t)r] + lam * cr[(size_t)r];
                for (int k = 1; k < K; ++k) {
                    const double j = cd[(size_t)(k * rows + r)] + lam * cr[(size_t)(k * rows + r)];
                    if (j < jbest) {
                        jbest = j;
                        best = k;
                    }
                }
                sel[(size_t)r] = best;
                rsel[(size_t)r] = cr[(size_t)(best * rows + r)];
            }
        });
        double total = 0.0;
        for (int64_t r = 0; r < rows; ++r) total += rsel[(size_t)r];
        if (it < 64) {
            if (total <= budget) hi = t;
            else lo = t;
        }
    }
}

int64_t tile_symbols_for(double target) {
    if (target <= 2.5) return 32768;
    if (target <= 5.0) return 16384;
    if (target <= 7.0) return 8192;
    return 4096;
}

void put32(uint8_t* p, uint32_t v) { std::memcpy(p, &v, 4); }  // little-endian hosts only
void put64(uint8_t* p, uint64_t v) { std::memcpy(p, &v, 8); }

std::vector<int64_t> sample_rows(int64_t rows, int64_t cols, const ep_encode_opts& o) {
    // sampled rows: partial Fisher-Yates driven by splitmix64 (Steele, Lea & Flood)
    const int64_t nq = (cols + 7) / 8;
    const int64_t sv = o.sample_vectors > 0 ? o.sample_vectors : (int64_t)1 << 18;
    const int64_t rs = std::max<int64_t>(1, std::min<int64_t>(rows, (sv + nq - 1) / nq));
    std::vector<int64_t> perm(rows);
    for (int64_t i = 0; i < rows; ++i) perm[i] = i;
    uint64_t st = o.seed ? o.seed : (((uint64_t)rows << 32) ^ (uint64_t)cols);
    std::vector<int64_t> srows(rs);
    for (int64_t i = 0; i < rs; ++i) {
        st += 0x9E3779B97F4A7C15ull;
        uint64_t z = st;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        z ^= z >> 31;
        const int64_t j = i + (int64_t)(z % (uint64_t)(rows - i));
        std::swap(perm[i], perm[j]);
        srows[i] = perm[i];
    }
    return srows;
}

int64_t side_bytes(const Hist& al, int64_t ntiles, int64_t rows, bool container) {
    int64_t tb = table_header_bytes(kTables);
    for (int t = 0; t < kTables; ++t) tb += 2 * (int64_t)al.alpha(t);
    int64_t side = tb + ntiles * (4 * kLanes + 4) + 4 + 4 * rows;
    if (container) side += 4 * rows;
    return side;
}

double estimate_bpp(Table* tabs, const Hist& al, int b, int64_t nvec, int64_t ns, int64_t ntiles, int64_t rows,
                    int64_t cols, bool container) {
    double bits = 0.0;
    for (int t = 0; t < kTables; ++t) {
        normalise(tabs[t], b);
        for (uint32_t k = 0; k < tabs[t].A; ++k)
            if (tabs[t].count[k]) bits += (double)tabs[t].count[k] * ((double)b - std::log2((double)tabs[t].freq[k]));
    }
    const double payload = bits / 8.0 * ((double)nvec / (double)ns);
    const double total = payload + (double)side_bytes(al, ntiles, rows, container);
    return 8.0 * total / (double)(rows * cols);  // per real weight
}

ep_blob* new_blob(int64_t rows, int64_t cols, int b, int64_t V, int64_t T, uint64_t words, const Table* tabs) {
    ep_blob* bl = (ep_blob*)std::calloc(1, sizeof(ep_blob));
    if (!bl) return nullptr;
    bl->rows = rows;
    bl->cols = cols;
    bl->b = b;
    bl->V = (int)V;
    bl->J = kLanes;
    bl->ntiles = (int)T;
    bl->payload_words = words;
    bl->payload_alloc_words = (words + 7) / 8 * 8;
    // the caller writes words [0, words); only the padding up to a multiple of 8 words is zeroed here
    const size_t alloc_words = std::max<size_t>(bl->payload_alloc_words, 8);
    bl->payload = (uint16_t*)std::malloc(alloc_words * sizeof(uint16_t));
    if (bl->payload) std::memset(bl->payload + words, 0, (alloc_words - words) * sizeof(uint16_t));
    bl->tile_index = (uint32_t*)std::malloc(sizeof(uint32_t) * (size_t)(kTileWords * T + 1));
    bl->freq_bytes = table_bytes(tabs);
    bl->freq_tables = (uint8_t*)std::calloc(bl->freq_bytes, 1);
    bl->row_scales = (float*)std::malloc(sizeof(float) * (size_t)rows);
    if (!bl->payload || !bl->tile_index || !bl->freq_tables || !bl->row_scales) {
        ep_free_blob(bl);
        return nullptr;
    }
    write_tables(bl->freq_tables, rows, cols, b, V, T, tabs);
    return bl;
}

size_t table_bytes(const Table* tabs) {
    int64_t nf = 0;
    for (int t = 0; t < kTables; ++t) nf += tabs[t].A;
    return (size_t)(table_header_bytes(kTables) + 2 * nf);
}

void write_tables(uint8_t* h, int64_t rows, int64_t cols, int b, int64_t V, int64_t T, const Table* tabs) {
    put32(h + 0, kMagic);
    put32(h + 4, kVersion);
    put32(h + 8, (uint32_t)b);
    put32(h + 12, (uint32_t)V);
    put32(h + 16, (uint32_t)kLanes);
    put32(h + 20, (uint32_t)T);
    put64(h + 24, (uint64_t)rows);
    put64(h + 32, (uint64_t)cols);
    put32(h + 40, (uint32_t)kTables);
    put32(h + 44, 0u);
    int64_t fo = table_header_bytes(kTables);
    for (int t = 0; t < kTables; ++t) {
        put32(h + kHeaderFixedBytes + 8 * t, (uint32_t)tabs[t].min);
        put32(h + kHeaderFixedBytes + 8 * t + 4, tabs[t].A);
        for (uint32_t k = 0; k < tabs[t].A; ++k) {
            const uint16_t v = (uint16_t)tabs[t].freq[k];
            std::memcpy(h + fo, &v, 2);
            fo += 2;
        }
    }
}

int64_t stored_bytes(uint64_t words, int64_t T, size_t freq_bytes, int64_t rows, bool container) {
    return (int64_t)(2 * words) + (int64_t)(4 * ((size_t)kTileWords * T + 1)) + (int64_t)freq_bytes + 4 * rows +
           (container ? 4 * rows : 0);
}

void finish_blob(ep_blob* bl, double s, bool container) {
    const int64_t rows = bl->rows;
    bl->s = s;
    bl->stored_bytes = stored_bytes(bl->payload_words, bl->ntiles, bl->freq_bytes, rows, container);
    bl->stored_bpp = 8.0 * (double)bl->stored_bytes / (double)(rows * bl->cols);
}

}  // namespace host
}  // namespace ep

extern "C" {

ep_status ep_encode_tensor(const float* W, int64_t rows, int64_t cols, double target_bpp, const ep_encode_opts* opts,
                           ep_blob** out) {
    using namespace ep;
    if (!W || !out) return EP_EINVAL;
    *out = nullptr;
    if (rows <= 0 || cols <= 0 || !(target_bpp > 0.0)) return EP_EINVAL;
    ep_encode_opts o{};
    if (opts) o = *opts;
    int b = o.prob_bits > 0 ? o.prob_bits : (target_bpp <= 7.0 ? 11 : 12);
    if (b < kMinB || b > kMaxB) return EP_EINVAL;
    const int64_t nq = (cols + 7) / 8, nvec = rows * nq;  // rows padded to whole vectors
    if (nvec >= (1ll << 31)) return EP_EINVAL;
    const int64_t V = o.tile_vectors > 0 ? o.tile_vectors : std::max<int64_t>(32, tile_symbols_for(target_bpp) / 9);
    int nthreads = o.num_threads > 0 ? o.num_threads : (int)std::max(1u, std::thread::hardware_concurrency());

    try {
        Encoder enc;
        enc.W = W;
        enc.rows = rows;
        enc.cols = cols;
        enc.nq = nq;
        enc.nvec = nvec;
        enc.target = target_bpp;
        enc.nthreads = nthreads;
        enc.container = o.has_container_scales != 0;
        enc.ntiles = (nvec + V - 1) / V;
        if (enc.ntiles >= (1ll << 31) / kTileWords) return EP_EINVAL;

        // row normalisation: RMS of the row, 1 for an all-zero row
        enc.norms.resize(rows);
        parallel_for(rows, nthreads, [&](int64_t a, int64_t e) {
            for (int64_t r = a; r < e; ++r) {
                const float* w = W + r * cols;
                double acc = 0.0;
                for (int64_t j = 0; j < cols; ++j) acc += (double)w[j] * (double)w[j];
                const double n = std::sqrt(acc / (double)cols);
                enc.norms[r] = n > 0.0 ? n : 1.0;
            }
        });

        const std::vector<int64_t> srows = host::sample_rows(rows, cols, o);
        const int64_t rs = (int64_t)srows.size();
        std::vector<int32_t> sf((size_t)(kFields * nq * rs));
        std::vector<int32_t> fields((size_t)(kFields * nvec));
        std::vector<double> num(rows), den(rows);

        auto quantize_all = [&](double s) {
            parallel_for(rows, nthreads, [&](int64_t a, int64_t e) {
                for (int64_t r = a; r < e; ++r)
                    quantize_row(W + r * cols, cols, enc.norms[r], s, fields.data() + (size_t)(kFields * nq * r),
                                 &num[r], &den[r]);
            });
        };

        const int steps = o.search_steps > 0 ? o.search_steps : 12;
        double s = 1.0;
        Hist al;
        for (;;) {
            double lo = 1e-3, hi = 8.0;
            for (int it = 0; it < steps; ++it) {
                s = std::sqrt(lo * hi);
                if (enc.estimate(srows, s, b, sf) > target_bpp) lo = s;
                else hi = s;
            }
            s = std::sqrt(lo * hi);
            quantize_all(s);
            al = alphabet_of(fields.data(), nvec, nthreads);
            if (al.amax_coord() <= (1ull << b)) break;
            if (b < kMaxB) {
                ++b;
                continue;
            }
            while (al.amax_coord() > (1ull << b)) {
                s = 1.05 * s * (double)al.amax_coord() / (double)(1u << b);
                quantize_all(s);
                al = alphabet_of(fields.data(), nvec, nthreads);
            }
            break;
        }
        std::vector<float> scales(rows);
        for (int64_t r = 0; r < rows; ++r) scales[r] = den[r] == 0.0 ? 0.0f : (float)(num[r] / den[r]);
        if (o.rdo_candidates > 1) {
            rdo_refine(W, rows, cols, enc.norms, s, b, o.rdo_candidates, o.rdo_sweeps > 0 ? o.rdo_sweeps : 1,
                       nthreads, fields, scales);
            al = alphabet_of(fields.data(), nvec, nthreads);
        }

        Table tabs[kTables];
        count_fields(fields.data(), nvec, al, tabs, nthreads);
        for (int t = 0; t < kTables; ++t) {
            if (tabs[t].A > (1u << b)) return EP_EALPHABET;
            normalise(tabs[t], b);
        }

        // tiles in parallel, then concatenated
        const int64_t T = enc.ntiles;
        std::vector<std::vector<uint16_t>> tile_words(T);
        std::vector<uint32_t> tix((size_t)(kTileWords * T + 1), 0);
        parallel_for(T, nthreads, [&](int64_t a, int64_t e) {
            for (int64_t t = a; t < e; ++t) {
                const int64_t v0 = t * V;
                const int64_t vt = std::min<int64_t>(V, nvec - v0);
                encode_tile(fields.data(), v0, vt, tabs, b, tile_words[t], tix.data() + kTileWords * t + 1);
            }
        });
        uint64_t words = 0;
        for (int64_t t = 0; t < T; ++t) {
            if (words >= 0xFFFFFFFFull) return EP_EINVAL;
            tix[kTileWords * t] = (uint32_t)words;
            words += tile_words[t].size();
        }
        if (words > 0xFFFFFFFFull) return EP_EINVAL;
        tix[kTileWords * T] = (uint32_t)words;

        ep_blob* bl = host::new_blob(rows, cols, b, V, T, words, tabs);
        if (!bl) return EP_ENOMEM;
        size_t o16 = 0;
        for (int64_t t = 0; t < T; ++t) {
            if (!tile_words[t].empty())
                std::memcpy(bl->payload + o16, tile_words[t].data(), 2 * tile_words[t].size());
            o16 += tile_words[t].size();
        }
        std::memcpy(bl->tile_index, tix.data(), sizeof(uint32_t) * tix.size());
        std::memcpy(bl->row_scales, scales.data(), sizeof(float) * (size_t)rows);
        host::finish_blob(bl, s, enc.container);
        *out = bl;
        return EP_OK;
    } catch (const std::bad_alloc&) {
        return EP_ENOMEM;
    }
}

void ep_free_blob(ep_blob* bl) {
    if (!bl) return;
    std::free(bl->payload);
    std::free(bl->tile_index);
    std::free(bl->freq_tables);
    std::free(bl->row_scales);
    std::free(bl);
}

}  // extern "C"
