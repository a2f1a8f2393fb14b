// encode_host.h -- host-side pieces both packers share (the CPU packer in encode.cpp and the
// GPU encoder in encode_gpu.cu): symbol ranges and counts of the 17 tables, their
// normalisation to 2^b, the sampled rows of the scale search, the stored-size estimate
// from counted tables, and the blob assembly.  Library-internal.
#pragma once

#include <algorithm>
#include <cstdint>
#include <vector>

#include "entropack.h"
#include "ep_format.h"

namespace ep {
namespace host {

// [min, max] of every table's symbols
struct Hist {
    int64_t lo[kTables], hi[kTables];
    void reset() {
        for (int t = 0; t < kTables; ++t) {
            lo[t] = INT64_MAX;
            hi[t] = INT64_MIN;
        }
    }
    void add_range(const int32_t* f, int64_t n) {
        for (int64_t g = 0; g < n; ++g) {
            const int32_t* v = f + kFields * g;
            for (int k = 0; k < kFields; ++k) {
                const int t = table_index(k, v[0]);
                lo[t] = std::min<int64_t>(lo[t], v[k]);
                hi[t] = std::max<int64_t>(hi[t], v[k]);
            }
        }
    }
    void merge(const Hist& o) {
        for (int t = 0; t < kTables; ++t) {
            lo[t] = std::min(lo[t], o.lo[t]);
            hi[t] = std::max(hi[t], o.hi[t]);
        }
    }
    uint64_t alpha(int t) const { return hi[t] >= lo[t] ? (uint64_t)(hi[t] - lo[t] + 1) : 0; }
    uint64_t amax_coord() const {
        uint64_t m = 0;
        for (int t = 1; t < kTables; ++t) m = std::max(m, alpha(t));
        return m;
    }
};

struct Table {
    int32_t min = 0;
    uint32_t A = 0;
    uint64_t total = 0;
    std::vector<uint64_t> count;
    std::vector<uint32_t> freq, cum;
};

// Frequencies at 2^b from counts (fills freq and cum).
void normalise(Table& tb, int b);
// The per-row refinement's K candidate ratios (App. C.2), nested in K (K <= 64).
void rdo_ratios(int K, double* rho);
// The refinement's selection (App. C.2): bisect log2 lambda on [-80, 80] (64 steps) for the smallest
// lambda whose per-row choices argmin_k cd[k][r] + lambda cr[k][r] (ties: lowest k; arrays k-major,
// rows per candidate) have total rate <= budget; the last lambda's choices into sel[rows].
void rdo_bisect(const double* cd, const double* cr, int64_t rows, int K, double budget, int nthreads, int* sel);
// S of the pages' tile sizing for a target rate (V = max(32, S / 9)).
int64_t tile_symbols_for(double target);
// The rows of the scale search's sample, in sample order.
std::vector<int64_t> sample_rows(int64_t rows, int64_t cols, const ep_encode_opts& o);
// Stored bytes other than the payload: tables, tile records, row scales (and container scales).
int64_t side_bytes(const Hist& al, int64_t ntiles, int64_t rows, bool container);
// Stored bits per real weight estimated from the sample's counted tables (normalises them):
// ideal code length of the ns sampled vectors scaled to nvec, plus side_bytes.
double estimate_bpp(Table* tabs, const Hist& al, int b, int64_t nvec, int64_t ns, int64_t ntiles, int64_t rows,
                    int64_t cols, bool container);
// A blob with its header and tables written and its payload (rounded up to 8 words, the words
// past `words` zeroed), tile index and row scales allocated for the caller to fill; nullptr
// when out of memory.
ep_blob* new_blob(int64_t rows, int64_t cols, int b, int64_t V, int64_t T, uint64_t words, const Table* tabs);
// Bytes of the table header and frequencies, and their writer (into a zeroed buffer of that size).
size_t table_bytes(const Table* tabs);
void write_tables(uint8_t* h, int64_t rows, int64_t cols, int b, int64_t V, int64_t T, const Table* tabs);
// Stored bytes of a stream: payload, tile records, tables, row scales (and container scales).
int64_t stored_bytes(uint64_t words, int64_t T, size_t freq_bytes, int64_t rows, bool container);
// Stored bytes and bits per weight of a filled blob.
void finish_blob(ep_blob* bl, double s, bool container);

}  // namespace host
}  // namespace ep
