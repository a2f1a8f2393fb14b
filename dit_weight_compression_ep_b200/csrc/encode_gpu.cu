// encode_gpu.cu -- ep_encode_tensor_gpu (host blob out) and ep_encode_tensor_gpu_device
// (device blob out; float32 or bfloat16 in): the packer with its full-tensor stages on the GPU.
//
// EntroPack paper §3.1 pipeline, as in encode.cpp: row normalisation, the sampled-row scale
// search (§3.4, App. C.1), full-tensor E8 quantisation (§1, Conway & Sloane 1982), the row-scale
// refit (§3.5), the seventeen coset-conditioned tables (§3.6, App. A.3) and tiled interleaved
// rANS (§3.6, App. C.3).  The result is byte for byte the CPU packer's blob:
//   - every floating-point step is the host's operation in the host's order (each row's sums
//     are taken in column order), and this file is compiled without
//     multiply-add contraction (-fmad=false), so each product and sum rounds as on the host;
//     division, square root and rint are IEEE round-to-nearest on both sides;
//   - the search's estimates come from exact integer counts made here and turned into bits on
//     the host by the same code as the CPU packer (normalisation and log2 stay on the host);
//   - the rANS step is integer arithmetic; a warp encodes a tile, lane j holding the tile's
//     lane j, and each step's words are placed in the order the host emits them.
// What runs on the host: the sample choice, the search's decisions, the b escalation, table
// normalisation, the per-row refinement's lambda bisection (App. C.2) and the blob header.

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <mutex>
#include <new>
#include <thread>
#include <vector>

#include "encode_host.h"
#include "entropack.h"
#include "ep_format.h"

namespace ep {
namespace {

using host::Hist;
using host::Table;

constexpr int kQThreads = 256;

// ------------------------------------------------------------ the quantiser

// Nearest point of D8: round to nearest (ties to even); an odd sum moves the coordinate
// furthest from its rounding (the first such) one step the other way (up when u - a >= 0).
__device__ __forceinline__ void d8_nearest(const double (&u)[8], double (&a)[8]) {
    long long par = 0;
    int far_k = 0;
    double far_d = -1.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        a[k] = rint(u[k]);
        par += (long long)a[k];
        const double d = fabs(u[k] - a[k]);
        if (d > far_d) {
            far_d = d;
            far_k = k;
        }
    }
    if (par & 1LL) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k == far_k) a[k] += (u[k] - a[k] >= 0.0) ? 1.0 : -1.0;
    }
}

// E8 = D8 u (D8 + 1/2), the nearer coset (ties to D8); the fields (c, z1..z7, m) into f.
__device__ __forceinline__ void e8_fields(const double (&u)[8], int32_t* f) {
    double a[8], h[8], v[8];
    d8_nearest(u, a);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = u[k] - 0.5;
    d8_nearest(v, h);
    double da = 0.0, dh = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const double ea = u[k] - a[k];
        const double eh = u[k] - (h[k] + 0.5);
        da += ea * ea;
        dh += eh * eh;
    }
    const int c = dh < da ? 1 : 0;
    long long s7 = 0;
    f[0] = c;
#pragma unroll
    for (int k = 0; k < 7; ++k) {
        const double z = c ? h[k] : a[k];
        f[1 + k] = (int32_t)z;
        s7 += (long long)z;
    }
    const long long z8 = (long long)(c ? h[7] : a[7]);
    f[8] = (int32_t)((z8 - (s7 & 1LL)) / 2);
}

// ----------------------------------------------------------------- kernels

// Per-row sums in column order: a warp owns 32 rows (lane i adds row r0 + i, so every row's sum
// is the host's sequential sum).  Columns go in chunks of 32, copied (lane = column, coalesced)
// by cp.async into a ring of shared-memory slots kept kDepth chunks ahead, so the loads stay in
// flight without holding registers while each lane adds its row's 32 entries from the slot.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Row normaliser: the RMS of the row (a sum of squares in index order), 1 for a zero row.
constexpr int kNormDepth = 8;
__global__ void __launch_bounds__(32) k_norms(const float* W, int64_t rows, int64_t cols, double* norms) {
    __shared__ float ring[kNormDepth][32][33];
    const int lane = threadIdx.x & 31;
    const int64_t r0 = (int64_t)blockIdx.x * 32;
    const int nr = rows - r0 < 32 ? (int)(rows - r0) : 32;
    const int64_t nch = (cols + 31) / 32;
    auto issue = [&](int64_t c) {
        if (c < nch) {
            const int64_t col = 32 * c + lane;
            if (col < cols)
                for (int rr = 0; rr < nr; ++rr) cp_async4(&ring[c % kNormDepth][rr][lane], W + (r0 + rr) * cols + col);
        }
        cp_async_commit();  // an empty group past the end keeps the group count in step
    };
    for (int64_t c = 0; c < kNormDepth - 1; ++c) issue(c);
    double acc = 0.0;
    for (int64_t c = 0; c < nch; ++c) {
        issue(c + kNormDepth - 1);
        cp_async_wait<kNormDepth - 1>();  // chunk c has landed (this lane's copies)
        __syncwarp();                     // and every lane's
        const int n = cols - 32 * c < 32 ? (int)(cols - 32 * c) : 32;
        const float* src = &ring[c % kNormDepth][lane][0];
        for (int k = 0; k < n; ++k) {
            const double w = (double)src[k];
            acc += w * w;
        }
        __syncwarp();  // the slot is refilled by the next iteration's copies
    }
    cp_async_wait<0>();
    if (lane < nr) {
        const double n = sqrt(acc / (double)cols);
        norms[r0 + lane] = n > 0.0 ? n : 1.0;
    }
}

// Fields of vectors [0, nrows * nq) at scale s: vector (i, q) is vector q of row rowlist[i]
// (row i without a list); a partial last vector is padded with zeros.
__global__ void k_quantize(const float* W, int64_t cols, int64_t nq, const double* norms, const int64_t* rowlist,
                           int64_t nrows, double s, int32_t* fields) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= nrows * nq) return;
    const int64_t i = g / nq, q = g - i * nq;
    const int64_t r = rowlist ? rowlist[i] : i;
    const float* w = W + r * cols + 8 * q;
    const double n = norms[r];
    const int64_t real = cols - 8 * q < 8 ? cols - 8 * q : 8;
    double u[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) u[k] = k < real ? ((double)w[k] / n) / s : 0.0;
    e8_fields(u, fields + kFields * g);
}

// [min, max] of every table's symbols over vectors [0, nvec) (lohi: 17 minima, then 17 maxima).
constexpr int kAlphaWarps = 8;
__global__ void __launch_bounds__(32 * kAlphaWarps) k_alphabet(const int32_t* fields, int64_t nvec, int* lohi) {
    int lo[kTables], hi[kTables];
#pragma unroll
    for (int t = 0; t < kTables; ++t) {
        lo[t] = INT_MAX;
        hi[t] = INT_MIN;
    }
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nvec; g += (int64_t)gridDim.x * blockDim.x) {
        const int32_t* v = fields + kFields * g;
        const int c = v[0];
        lo[0] = min(lo[0], c);
        hi[0] = max(hi[0], c);
#pragma unroll
        for (int k = 1; k < kFields; ++k) {
            const int x = v[k];
            // table 1 + 2(k - 1) + c, written without a dynamic index
            if (c) {
                lo[2 * k] = min(lo[2 * k], x);
                hi[2 * k] = max(hi[2 * k], x);
            } else {
                lo[2 * k - 1] = min(lo[2 * k - 1], x);
                hi[2 * k - 1] = max(hi[2 * k - 1], x);
            }
        }
    }
    // warp, then block, then one atomic per table per block (the 34 words are shared by every block)
    __shared__ int part[kAlphaWarps][2 * kTables];
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int t = 0; t < kTables; ++t) {
        int a = lo[t], b = hi[t];
        for (int o = 16; o > 0; o >>= 1) {
            a = min(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
            b = max(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
        }
        if (lane == 0) {
            part[wid][t] = a;
            part[wid][kTables + t] = b;
        }
    }
    __syncthreads();
    if (threadIdx.x < 2 * kTables) {
        const int i = threadIdx.x;
        int v = part[0][i];
        for (int w = 1; w < kAlphaWarps; ++w) v = i < kTables ? min(v, part[w][i]) : max(v, part[w][i]);
        if (i < kTables && v != INT_MAX) atomicMin(lohi + i, v);
        if (i >= kTables && v != INT_MIN) atomicMax(lohi + i, v);
    }
}

// Counts of every table's symbols over vectors [0, nvec): per-CTA shared histograms (dynamic
// shared memory, nbins words) when the tables' bins fit (nbins <= kSmemBins: up to 224 KiB, which
// holds the alphabets of b <= 12 at high rates), global atomics otherwise.
constexpr int kSmemBins = 56 * 1024;
struct CountArgs {
    int tmin[kTables];
    uint32_t tbase[kTables];
};
__global__ void k_count(const int32_t* fields, int64_t nvec, CountArgs ca, uint32_t nbins, unsigned long long* counts) {
    extern __shared__ uint32_t sh[];
    const bool in_smem = nbins <= (uint32_t)kSmemBins;
    if (in_smem)
        for (uint32_t i = threadIdx.x; i < nbins; i += blockDim.x) sh[i] = 0;
    __syncthreads();
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nvec; g += (int64_t)gridDim.x * blockDim.x) {
        const int32_t* v = fields + kFields * g;
        const int c = v[0];
#pragma unroll
        for (int k = 0; k < kFields; ++k) {
            const int t = table_index(k, c);
            const uint32_t bin = ca.tbase[t] + (uint32_t)(v[k] - ca.tmin[t]);
            if (in_smem) atomicAdd(sh + bin, 1u);
            else atomicAdd(counts + bin, 1ull);
        }
    }
    if (in_smem) {
        __syncthreads();
        for (uint32_t i = threadIdx.x; i < nbins; i += blockDim.x)
            if (sh[i]) atomicAdd(counts + i, (unsigned long long)sh[i]);
    }
}

// Row scales: the least-squares scale <w, y> / <y, y> over the real entries, sums in index
// order (y = z + c/2 rebuilt from the fields), 0 for a zero denominator.  DIST: instead, the
// distortion sum (w - sigma y)^2 in index order with sigma = sg_in[row] (the refinement's
// candidates, App. C.2).  Same ring as k_norms, with the fields of the chunk's four vectors
// (36 words a row) beside its 32 weights.
constexpr int kRefitDepth = 4;
template <bool DIST>
__global__ void __launch_bounds__(32) k_rowpass(const float* W, int64_t rows, int64_t cols, int64_t nq,
                                                 const int32_t* fields, const float* sg_in, float* scales,
                                                 double* dist) {
    __shared__ float rw[kRefitDepth][32][33];
    __shared__ int32_t rf[kRefitDepth][32][37];
    const int lane = threadIdx.x & 31;
    const int64_t r0 = (int64_t)blockIdx.x * 32;
    const int nr = rows - r0 < 32 ? (int)(rows - r0) : 32;
    const int64_t nch = (cols + 31) / 32;
    auto issue = [&](int64_t c) {
        if (c < nch) {
            const int slot = (int)(c % kRefitDepth);
            const int64_t col = 32 * c + lane;
            const int64_t nv = nq - 4 * c < 4 ? nq - 4 * c : 4;  // vectors of this chunk
            for (int rr = 0; rr < nr; ++rr) {
                if (col < cols) cp_async4(&rw[slot][rr][lane], W + (r0 + rr) * cols + col);
                const int32_t* f = fields + kFields * ((r0 + rr) * nq + 4 * c);
                if (lane < kFields * nv) cp_async4(&rf[slot][rr][lane], f + lane);
                if (lane + 32 < kFields * nv) cp_async4(&rf[slot][rr][lane + 32], f + lane + 32);
            }
        }
        cp_async_commit();
    };
    for (int64_t c = 0; c < kRefitDepth - 1; ++c) issue(c);
    double sn = 0.0, sd = 0.0;
    const double sg = DIST && lane < nr ? (double)sg_in[r0 + lane] : 0.0;
    for (int64_t c = 0; c < nch; ++c) {
        issue(c + kRefitDepth - 1);
        cp_async_wait<kRefitDepth - 1>();
        __syncwarp();
        const int slot = (int)(c % kRefitDepth);
        const int n = cols - 32 * c < 32 ? (int)(cols - 32 * c) : 32;
        const float* w = &rw[slot][lane][0];
        const int32_t* f = &rf[slot][lane][0];
        for (int k0 = 0; k0 < n && lane < nr; k0 += 8) {  // (lanes past the last row add nothing)
            const int32_t* v = f + kFields * (k0 >> 3);
            const double half_c = 0.5 * v[0];
            long long s7 = 0;
            for (int k = 0; k < 7; ++k) s7 += v[1 + k];
            const int m = n - k0 < 8 ? n - k0 : 8;
            for (int k = 0; k < m; ++k) {
                const long long z = k < 7 ? (long long)v[1 + k] : 2LL * v[8] + (s7 & 1LL);
                const double y = (double)z + half_c;
                if constexpr (DIST) {
                    const double er = (double)w[k0 + k] - sg * y;
                    sn += er * er;
                } else {
                    sn += (double)w[k0 + k] * y;
                    sd += y * y;
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    if (lane < nr) {
        if constexpr (DIST) dist[r0 + lane] = sn;
        else scales[r0 + lane] = sd == 0.0 ? 0.0f : (float)(sn / sd);
    }
}

// The refinement's admissibility: a row's candidate is admissible when every symbol lies in the
// baseline tables' alphabets (ok[row] cleared otherwise; the caller sets it to 1 first).
struct AlphaArgs {
    int tmin[kTables];
    uint32_t A[kTables];
};
__global__ void k_admissible(const int32_t* fields, int64_t nvec, int64_t nq, AlphaArgs aa, uint8_t* ok) {
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nvec; g += (int64_t)gridDim.x * blockDim.x) {
        const int32_t* v = fields + kFields * g;
        bool in = true;
#pragma unroll
        for (int m = 0; m < kFields; ++m) {
            const int t = table_index(m, v[0] & 1);
            const int64_t i = (int64_t)v[m] - aa.tmin[t];
            in = in && aa.A[t] != 0 && i >= 0 && i < (int64_t)aa.A[t];
        }
        if (!in) ok[g / nq] = 0;
    }
}

// A row's ideal code length under tables (the refinement's rate): the cost of every symbol, in
// vector and field order, summed in that order; cost = b - log2 f from a host-made table, b for
// a symbol the tables give no frequency.  Same ring as k_rowpass, fields only.
struct CostArgs {
    int tmin[kTables];
    uint32_t A[kTables];
    uint32_t base[kTables];
    double b;
    const double* cost;
};
__global__ void __launch_bounds__(32) k_row_bits(const int32_t* fields, int64_t rows, int64_t nq, CostArgs ca,
                                                  double* bits) {
    __shared__ int32_t rf[kRefitDepth][32][37];
    const int lane = threadIdx.x & 31;
    const int64_t r0 = (int64_t)blockIdx.x * 32;
    const int nr = rows - r0 < 32 ? (int)(rows - r0) : 32;
    const int64_t nch = (nq + 3) / 4;
    auto issue = [&](int64_t c) {
        if (c < nch) {
            const int slot = (int)(c % kRefitDepth);
            const int64_t nv = nq - 4 * c < 4 ? nq - 4 * c : 4;
            for (int rr = 0; rr < nr; ++rr) {
                const int32_t* f = fields + kFields * ((r0 + rr) * nq + 4 * c);
                if (lane < kFields * nv) cp_async4(&rf[slot][rr][lane], f + lane);
                if (lane + 32 < kFields * nv) cp_async4(&rf[slot][rr][lane + 32], f + lane + 32);
            }
        }
        cp_async_commit();
    };
    for (int64_t c = 0; c < kRefitDepth - 1; ++c) issue(c);
    double acc = 0.0;
    for (int64_t c = 0; c < nch; ++c) {
        issue(c + kRefitDepth - 1);
        cp_async_wait<kRefitDepth - 1>();
        __syncwarp();
        const int nv = nq - 4 * c < 4 ? (int)(nq - 4 * c) : 4;
        const int32_t* f = &rf[(int)(c % kRefitDepth)][lane][0];
        // lanes past the last row have no copies in the slot: they add nothing (their slots hold
        // stale words, which must not index the tables)
        for (int q = 0; q < nv && lane < nr; ++q) {
            const int32_t* v = f + kFields * q;
            for (int m = 0; m < kFields; ++m) {
                const int t = table_index(m, v[0] & 1);
                const int64_t i = (int64_t)v[m] - ca.tmin[t];
                acc += (ca.A[t] != 0 && i >= 0 && i < (int64_t)ca.A[t]) ? ca.cost[ca.base[t] + (uint32_t)i] : ca.b;
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    if (lane < nr) bits[r0 + lane] = acc;
}

// fields[row] = candidate sel[row]'s fields of that row (candidates k-major, rows per candidate)
__global__ void k_gather(const int32_t* cf, const int* sel, int64_t rows, int64_t rowf, int32_t* fields) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * rowf; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / rowf;
        fields[i] = cf[(int64_t)sel[r] * rows * rowf + i];
    }
}

// rANS, one warp per tile: lane j encodes the tile's lane j (vectors 32 r + j), steps in
// reverse.  The host emits a step's words in descending lane order and reverses the whole
// tile at the end; here lane j's word of a step goes to position n + (emitting lanes above j)
// of the reversed stream, n the words emitted before the step (the copy-out reverses).
struct RansArgs {
    const uint32_t* freq;  // every table's frequencies, back to back from tbase
    const uint32_t* cum;
    int tmin[kTables];
    uint32_t tbase[kTables];
};
__global__ void k_rans(const int32_t* fields, int64_t nvec, int64_t V, int64_t T, int b, RansArgs ra,
                       uint16_t* scratch, uint32_t* nwords, uint32_t* states) {
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    const int j = threadIdx.x & 31;
    const uint32_t above = j == 31 ? 0u : (0xFFFFFFFFu << (j + 1));
    const int64_t v0 = t * V;
    const int64_t vt = nvec - v0 < V ? nvec - v0 : V;
    const int64_t rounds = (vt + kLanes - 1) / kLanes;
    uint16_t* out = scratch + (size_t)t * (size_t)(kFields * V);
    const uint32_t M = 1u << b;
    uint32_t x = kStateLow, n = 0;
    for (int64_t st = kFields * rounds - 1; st >= 0; --st) {
        const int64_t r = st / kFields;
        const int k = (int)(st - r * kFields);
        const int64_t v = kLanes * r + j;
        const bool act = v < vt;
        bool emit = false;
        uint32_t word = 0;
        if (act) {
            const int32_t* f = fields + kFields * (v0 + v);
            const int tb = table_index(k, f[0]);
            const uint32_t idx = ra.tbase[tb] + (uint32_t)(f[k] - ra.tmin[tb]);
            const uint32_t fr = ra.freq[idx], cm = ra.cum[idx];
            if (x >= (fr << (31 - b))) {
                emit = true;
                word = x & 0xFFFFu;
                x >>= 16;
            }
            x = (x / fr) * M + (x % fr) + cm;
        }
        const uint32_t em = __ballot_sync(0xFFFFFFFFu, emit);
        if (emit) out[n + __popc(em & above)] = (uint16_t)word;
        n += __popc(em);
    }
    states[(size_t)t * kLanes + j] = x;
    if (j == 0) nwords[t] = n;
}

// Tile t's words, reversed, to payload[off[t] ..).
__global__ void k_copy_out(const uint16_t* scratch, int64_t V, const uint32_t* nwords, const uint32_t* off,
                           uint16_t* payload) {
    const int64_t t = blockIdx.x;
    const uint32_t n = nwords[t];
    const uint16_t* src = scratch + (size_t)t * (size_t)(kFields * V);
    uint16_t* dst = payload + off[t];
    for (uint32_t i = threadIdx.x; i < n; i += blockDim.x) dst[i] = src[n - 1 - i];
}

// ------------------------------------------------------------- host side

// The encoder's scratch comes from a memory pool of the library's own, stream-ordered, which
// keeps up to kPoolKeep bytes between calls (no device-wide synchronisation per allocation).
constexpr uint64_t kPoolKeep = 1ull << 30;
std::mutex g_pool_mu;
cudaMemPool_t g_pool[64] = {};

cudaError_t pool_of(int dev, cudaMemPool_t& out) {
    std::lock_guard<std::mutex> lk(g_pool_mu);
    if (!g_pool[dev]) {
        cudaMemPoolProps pp = {};
        pp.allocType = cudaMemAllocationTypePinned;
        pp.location.type = cudaMemLocationTypeDevice;
        pp.location.id = dev;
        cudaError_t e = cudaMemPoolCreate(&g_pool[dev], &pp);
        if (e != cudaSuccess) return e;
        uint64_t keep = kPoolKeep;
        e = cudaMemPoolSetAttribute(g_pool[dev], cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) return e;
    }
    out = g_pool[dev];
    return cudaSuccess;
}

// A device buffer from the pool, released in stream order on every exit path.
struct DevBuf {
    void* p = nullptr;
    cudaStream_t st = nullptr;
    static thread_local cudaMemPool_t pool;  // the calling thread's device's pool, set per call
    ~DevBuf() {
        if (p) cudaFreeAsync(p, st);
    }
    template <typename T>
    T* as() const {
        return static_cast<T*>(p);
    }
    cudaError_t alloc(size_t bytes, cudaStream_t s) {
        st = s;
        return cudaMallocFromPoolAsync(&p, bytes > 0 ? bytes : 16, pool, s);
    }
};
thread_local cudaMemPool_t DevBuf::pool = nullptr;

__global__ void k_lohi_init(int* lohi) {
    const int t = threadIdx.x;
    if (t < kTables) {
        lohi[t] = INT_MAX;
        lohi[kTables + t] = INT_MIN;
    }
}

int grid_for(int64_t n, int threads) { return (int)std::max<int64_t>(1, (n + threads - 1) / threads); }

// the most bins a count needs: 16 coordinate tables of at most 2^15 symbols, the coset table's 2
constexpr uint32_t kMaxBins = 16u * 32768u + 2u;

struct GpuEncoder {
    cudaStream_t st;
    int nsm = 148;
    const float* W;
    int64_t rows, cols, nq, nvec;
    DevBuf d_lohi, d_counts;  // (the counts buffer holds kMaxBins)

    cudaError_t alphabet(const int32_t* f, int64_t n, Hist& al) {
        k_lohi_init<<<1, 32, 0, st>>>(d_lohi.as<int>());
        cudaError_t e;
        k_alphabet<<<std::min(grid_for(n, 32 * kAlphaWarps), 2 * nsm), 32 * kAlphaWarps, 0, st>>>(f, n,
                                                                                                 d_lohi.as<int>());
        int got[2 * kTables];
        e = cudaMemcpyAsync(got, d_lohi.p, sizeof(got), cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return e;
        al.reset();
        for (int t = 0; t < kTables; ++t) {
            if (got[t] == INT_MAX) continue;  // an empty table
            al.lo[t] = got[t];
            al.hi[t] = got[kTables + t];
        }
        return cudaSuccess;
    }

    // counts of vectors [0, n) into tables laid out like the CPU packer's count_fields
    cudaError_t count(const int32_t* f, int64_t n, const Hist& al, Table* tabs) {
        CountArgs ca;
        uint32_t nb = 0;
        for (int t = 0; t < kTables; ++t) {
            tabs[t].A = (uint32_t)al.alpha(t);
            tabs[t].min = tabs[t].A ? (int32_t)al.lo[t] : 0;
            tabs[t].total = 0;
            tabs[t].count.assign(std::max<uint32_t>(tabs[t].A, 1), 0);
            ca.tmin[t] = tabs[t].min;
            ca.tbase[t] = nb;
            nb += (uint32_t)tabs[t].count.size();
        }
        if (nb > kMaxBins) return cudaErrorInvalidValue;  // alphabets are checked against 2^b first
        cudaError_t e = cudaMemsetAsync(d_counts.p, 0, sizeof(unsigned long long) * nb, st);
        if (e != cudaSuccess) return e;
        const bool in_smem = nb <= (uint32_t)kSmemBins;
        const size_t smem = in_smem ? sizeof(uint32_t) * nb : 0;
        if (in_smem && smem > 48 * 1024) {
            e = cudaFuncSetAttribute(k_count, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(sizeof(uint32_t) * kSmemBins));
            if (e != cudaSuccess) return e;
        }
        // grid: as many CTAs as fit with that much shared memory (at least one per SM)
        const int per_sm = smem > 0 ? std::max(1, (int)((200 * 1024) / smem)) : 4;
        k_count<<<std::min(grid_for(n, 256), std::min(4, per_sm) * nsm), 256, smem, st>>>(
            f, n, ca, nb, d_counts.as<unsigned long long>());
        std::vector<unsigned long long> h(nb);
        e = cudaMemcpyAsync(h.data(), d_counts.p, sizeof(unsigned long long) * nb, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return e;
        for (int t = 0; t < kTables; ++t) {
            for (size_t s = 0; s < tabs[t].count.size(); ++s) {
                tabs[t].count[s] = h[ca.tbase[t] + s];
                tabs[t].total += h[ca.tbase[t] + s];
            }
        }
        return cudaSuccess;
    }

    cudaError_t quantize(const double* norms, const int64_t* rowlist, int64_t nr, double s, int32_t* f) {
        k_quantize<<<grid_for(nr * nq, kQThreads), kQThreads, 0, st>>>(W, cols, nq, norms, rowlist, nr, s, f);
        return cudaGetLastError();
    }
};

}  // namespace
}  // namespace ep

namespace ep {
namespace {

// bf16 weights widened to float32 (exact), so that both inputs run the same stages
__global__ void k_widen_bf16(const uint16_t* src, int64_t n, float* dst) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = __uint_as_float((uint32_t)src[i] << 16);
}

// Tile records [offset, state_0..31] and the final offset, from the offsets and states.
__global__ void k_tile_index(int64_t T, const uint32_t* off, const uint32_t* states, uint32_t total, uint32_t* tix) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i > kTileWords * T) return;
    const int64_t t = i / kTileWords, j = i - t * kTileWords;
    tix[i] = t == T ? total : (j == 0 ? off[t] : states[kLanes * t + (j - 1)]);
}

// Argument checks shared by both entry points; fills V and T.
ep_status check_encode_args(const void* W, int64_t rows, int64_t cols, double target_bpp, const ep_encode_opts& o,
                            int64_t& V, int64_t& T) {
    if (!W || rows <= 0 || cols <= 0 || !(target_bpp > 0.0)) return EP_EINVAL;
    const int b = o.prob_bits > 0 ? o.prob_bits : (target_bpp <= 7.0 ? 11 : 12);
    if (b < kMinB || b > kMaxB) return EP_EINVAL;
    const int64_t nq = (cols + 7) / 8, nvec = rows * nq;
    if (nvec >= (1ll << 31)) return EP_EINVAL;
    V = o.tile_vectors > 0 ? o.tile_vectors : std::max<int64_t>(32, host::tile_symbols_for(target_bpp) / 9);
    T = (nvec + V - 1) / V;
    if (T >= (1ll << 31) / kTileWords) return EP_EINVAL;
    return EP_OK;
}

// The current device, its SM count and its encoder pool; W checked to be memory it can read.
ep_status device_for(const void* W, int& dev, int& nsm) {
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return EP_ECUDA;
    // a host pointer would fault the first kernel
    cudaPointerAttributes pa = {};
    if (cudaPointerGetAttributes(&pa, W) != cudaSuccess) {
        cudaGetLastError();  // clear the error of an unknown pointer
        return EP_EINVAL;
    }
    if (!((pa.type == cudaMemoryTypeDevice && pa.device == dev) || pa.type == cudaMemoryTypeManaged)) return EP_EINVAL;
    return pool_of(dev, DevBuf::pool) == cudaSuccess ? EP_OK : EP_ECUDA;
}

// One encode's results, on the device in pool buffers (freed in stream order with it).
struct Encoded {
    DevBuf payload, scales, off, states;  // words, rows, T, 32 T
    uint64_t words = 0;
    int b = 0;
    double s = 0.0;
    Table tabs[kTables];
};

// The stages of ep_encode_tensor_gpu on float32 weights W (device) into `r`.
ep_status encode_core(cudaStream_t st, int nsm, const float* W, int64_t rows, int64_t cols, double target_bpp,
                      const ep_encode_opts& o, int64_t V, int64_t T, Encoded& r) {
    const int64_t nq = (cols + 7) / 8, nvec = rows * nq;
    const bool container = o.has_container_scales != 0;
    int b = o.prob_bits > 0 ? o.prob_bits : (target_bpp <= 7.0 ? 11 : 12);
    GpuEncoder g;
    g.st = st;
    g.nsm = nsm;
    g.W = W;
    g.rows = rows;
    g.cols = cols;
    g.nq = nq;
    g.nvec = nvec;
    DevBuf d_norms, d_srows, d_sf, d_fields;
    if (g.d_lohi.alloc(sizeof(int) * 2 * kTables, st) != cudaSuccess ||
        g.d_counts.alloc(sizeof(unsigned long long) * kMaxBins, st) || d_norms.alloc(sizeof(double) * rows, st) ||
        d_fields.alloc(sizeof(int32_t) * kFields * (size_t)nvec, st) || r.scales.alloc(sizeof(float) * rows, st))
        return EP_ECUDA;
    k_norms<<<grid_for(rows, 32), 32, 0, st>>>(W, rows, cols, d_norms.as<double>());

    const std::vector<int64_t> srows = host::sample_rows(rows, cols, o);
    const int64_t rs = (int64_t)srows.size(), ns = rs * nq;
    if (d_srows.alloc(sizeof(int64_t) * rs, st) || d_sf.alloc(sizeof(int32_t) * kFields * (size_t)ns, st))
        return EP_ECUDA;
    if (cudaMemcpyAsync(d_srows.p, srows.data(), sizeof(int64_t) * rs, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return EP_ECUDA;

    auto estimate = [&](double s, double& est) -> cudaError_t {
        cudaError_t e = g.quantize(d_norms.as<double>(), d_srows.as<int64_t>(), rs, s, d_sf.as<int32_t>());
        Hist al;
        if (e == cudaSuccess) e = g.alphabet(d_sf.as<int32_t>(), ns, al);
        if (e != cudaSuccess) return e;
        if (al.amax_coord() > (1ull << b)) {
            est = INFINITY;
            return cudaSuccess;
        }
        Table tabs[kTables];
        e = g.count(d_sf.as<int32_t>(), ns, al, tabs);
        if (e == cudaSuccess) est = host::estimate_bpp(tabs, al, b, nvec, ns, T, rows, cols, container);
        return e;
    };
    auto quantize_all = [&](double s, Hist& al) -> cudaError_t {
        cudaError_t e = g.quantize(d_norms.as<double>(), nullptr, rows, s, d_fields.as<int32_t>());
        return e == cudaSuccess ? g.alphabet(d_fields.as<int32_t>(), nvec, al) : e;
    };

    // the scale search and the b escalation, decided on the host as in the CPU packer
    const int steps = o.search_steps > 0 ? o.search_steps : 12;
    double s = 1.0;
    Hist al;
    for (;;) {
        double lo = 1e-3, hi = 8.0;
        for (int it = 0; it < steps; ++it) {
            s = std::sqrt(lo * hi);
            double est = 0.0;
            if (estimate(s, est) != cudaSuccess) return EP_ECUDA;
            if (est > target_bpp) lo = s;
            else hi = s;
        }
        s = std::sqrt(lo * hi);
        if (quantize_all(s, al) != cudaSuccess) return EP_ECUDA;
        if (al.amax_coord() <= (1ull << b)) break;
        if (b < kMaxB) {
            ++b;
            continue;
        }
        while (al.amax_coord() > (1ull << b)) {
            s = 1.05 * s * (double)al.amax_coord() / (double)(1u << b);
            if (quantize_all(s, al) != cudaSuccess) return EP_ECUDA;
        }
        break;
    }
    k_rowpass<false><<<grid_for(rows, 32), 32, 0, st>>>(W, rows, cols, nq, d_fields.as<int32_t>(), nullptr,
                                                        r.scales.as<float>(), nullptr);

    if (o.rdo_candidates > 1) {
        // App. C.2, as the CPU packer's rdo_refine: candidates at rho_k s, each refitted, its
        // distortion and admissibility; the rates priced under the current tables; the lambda
        // bisection and the selection on the host (host::rdo_bisect); the tables rebuilt
        const int K = o.rdo_candidates < 64 ? o.rdo_candidates : 64;
        const int sweeps = o.rdo_sweeps > 0 ? o.rdo_sweeps : 1;
        const int64_t rowf = kFields * nq;
        double rho[64];
        host::rdo_ratios(K, rho);
        Table base[kTables];
        if (g.count(d_fields.as<int32_t>(), nvec, al, base) != cudaSuccess) return EP_ECUDA;
        for (int t = 0; t < kTables; ++t) host::normalise(base[t], b);
        DevBuf d_cf, d_cs, d_cd, d_cr, d_ok, d_sel;
        if (d_cf.alloc(sizeof(int32_t) * (size_t)K * (size_t)nvec * kFields, st) ||
            d_cs.alloc(sizeof(float) * (size_t)K * rows, st) || d_cd.alloc(sizeof(double) * (size_t)K * rows, st) ||
            d_cr.alloc(sizeof(double) * (size_t)K * rows, st) || d_ok.alloc((size_t)K * rows, st) ||
            d_sel.alloc(sizeof(int) * rows, st) || cudaMemsetAsync(d_ok.p, 1, (size_t)K * rows, st))
            return EP_ECUDA;
        AlphaArgs aa;
        for (int t = 0; t < kTables; ++t) {
            aa.tmin[t] = base[t].min;
            aa.A[t] = base[t].A;
        }
        auto cand = [&](int k) { return d_cf.as<int32_t>() + (size_t)k * (size_t)nvec * kFields; };
        for (int k = 0; k < K; ++k) {
            if (g.quantize(d_norms.as<double>(), nullptr, rows, rho[k] * s, cand(k)) != cudaSuccess) return EP_ECUDA;
            k_rowpass<false><<<grid_for(rows, 32), 32, 0, st>>>(W, rows, cols, nq, cand(k), nullptr,
                                                                d_cs.as<float>() + (size_t)k * rows, nullptr);
            k_rowpass<true><<<grid_for(rows, 32), 32, 0, st>>>(W, rows, cols, nq, cand(k),
                                                               d_cs.as<float>() + (size_t)k * rows, nullptr,
                                                               d_cd.as<double>() + (size_t)k * rows);
            k_admissible<<<std::min(grid_for(nvec, 256), 8 * nsm), 256, 0, st>>>(cand(k), nvec, nq, aa,
                                                                               d_ok.as<uint8_t>() + (size_t)k * rows);
        }
        // every candidate's rate under `tabs` into out[k * rows + r] (k < nk)
        auto price = [&](const Table* tabs, int nk, double* out) -> cudaError_t {
            CostArgs ca;
            std::vector<double> cost;
            for (int t = 0; t < kTables; ++t) {
                ca.tmin[t] = tabs[t].min;
                ca.A[t] = tabs[t].A;
                ca.base[t] = (uint32_t)cost.size();
                for (uint32_t i = 0; i < tabs[t].A; ++i) {
                    const uint32_t fr = tabs[t].freq[i];
                    cost.push_back((double)b - std::log2((double)(fr ? fr : 1u)));
                }
            }
            ca.b = (double)b;  // a symbol without a frequency: b - log2 1
            DevBuf d_cost;
            cudaError_t e = d_cost.alloc(sizeof(double) * std::max<size_t>(cost.size(), 1), st);
            if (e == cudaSuccess && !cost.empty())
                e = cudaMemcpyAsync(d_cost.p, cost.data(), sizeof(double) * cost.size(), cudaMemcpyHostToDevice, st);
            if (e != cudaSuccess) return e;
            ca.cost = d_cost.as<double>();
            for (int k = 0; k < nk; ++k)
                k_row_bits<<<grid_for(rows, 32), 32, 0, st>>>(cand(k), rows, nq, ca, d_cr.as<double>() + (size_t)k * rows);
            e = cudaMemcpyAsync(out, d_cr.p, sizeof(double) * (size_t)nk * rows, cudaMemcpyDeviceToHost, st);
            return e == cudaSuccess ? cudaStreamSynchronize(st) : e;
        };
        std::vector<double> cd((size_t)K * rows), cr((size_t)K * rows), rsel((size_t)rows);
        std::vector<uint8_t> ok((size_t)K * rows);
        std::vector<int> sel((size_t)rows, 0);
        if (price(base, 1, rsel.data()) != cudaSuccess) return EP_ECUDA;  // the baseline's ideal code length
        double budget = 0.0;
        for (int64_t rr = 0; rr < rows; ++rr) budget += rsel[(size_t)rr];
        if (cudaMemcpyAsync(cd.data(), d_cd.p, sizeof(double) * cd.size(), cudaMemcpyDeviceToHost, st) ||
            cudaMemcpyAsync(ok.data(), d_ok.p, ok.size(), cudaMemcpyDeviceToHost, st) || cudaStreamSynchronize(st))
            return EP_ECUDA;
        const int nthreads = (int)std::max(1u, std::thread::hardware_concurrency());
        Table next[kTables];
        const Table* model = base;
        for (int sw = 0; sw < sweeps; ++sw) {
            if (price(model, K, cr.data()) != cudaSuccess) return EP_ECUDA;
            for (size_t i = 0; i < cr.size(); ++i)
                if (!ok[i]) cr[i] = INFINITY;
            host::rdo_bisect(cd.data(), cr.data(), rows, K, budget, nthreads, sel.data());
            if (cudaMemcpyAsync(d_sel.p, sel.data(), sizeof(int) * rows, cudaMemcpyHostToDevice, st)) return EP_ECUDA;
            k_gather<<<std::min(grid_for(rows * rowf, 256), 16 * nsm), 256, 0, st>>>(d_cf.as<int32_t>(),
                                                                                   d_sel.as<int>(), rows, rowf,
                                                                                   d_fields.as<int32_t>());
            Hist aln;
            if (g.alphabet(d_fields.as<int32_t>(), nvec, aln) != cudaSuccess ||
                g.count(d_fields.as<int32_t>(), nvec, aln, next) != cudaSuccess)
                return EP_ECUDA;
            for (int t = 0; t < kTables; ++t) host::normalise(next[t], b);
            model = next;
        }
        // the chosen candidates' row scales
        std::vector<float> cs((size_t)K * rows), sc((size_t)rows);
        if (cudaMemcpyAsync(cs.data(), d_cs.p, sizeof(float) * cs.size(), cudaMemcpyDeviceToHost, st) ||
            cudaStreamSynchronize(st))
            return EP_ECUDA;
        for (int64_t rr = 0; rr < rows; ++rr) sc[(size_t)rr] = cs[(size_t)sel[(size_t)rr] * rows + rr];
        if (cudaMemcpyAsync(r.scales.p, sc.data(), sizeof(float) * rows, cudaMemcpyHostToDevice, st) ||
            g.alphabet(d_fields.as<int32_t>(), nvec, al) != cudaSuccess)
            return EP_ECUDA;
    }

    if (g.count(d_fields.as<int32_t>(), nvec, al, r.tabs) != cudaSuccess) return EP_ECUDA;
    for (int t = 0; t < kTables; ++t) {
        if (r.tabs[t].A > (1u << b)) return EP_EALPHABET;
        host::normalise(r.tabs[t], b);
    }

    // rANS: the tables to the device, a warp per tile into scratch, then the words in order
    RansArgs ra;
    std::vector<uint32_t> hf, hc;
    for (int t = 0; t < kTables; ++t) {
        ra.tmin[t] = r.tabs[t].min;
        ra.tbase[t] = (uint32_t)hf.size();
        for (size_t k = 0; k < r.tabs[t].freq.size(); ++k) {
            hf.push_back(r.tabs[t].freq[k]);
            hc.push_back(r.tabs[t].cum[k]);
        }
    }
    DevBuf d_freq, d_cum, d_scratch, d_nwords;
    if (d_freq.alloc(4 * hf.size(), st) || d_cum.alloc(4 * hc.size(), st) ||
        d_scratch.alloc(sizeof(uint16_t) * (size_t)kFields * (size_t)V * (size_t)T, st) ||
        d_nwords.alloc(4 * T, st) || r.states.alloc(sizeof(uint32_t) * kLanes * (size_t)T, st) ||
        r.off.alloc(4 * T, st))
        return EP_ECUDA;
    if (cudaMemcpyAsync(d_freq.p, hf.data(), 4 * hf.size(), cudaMemcpyHostToDevice, st) ||
        cudaMemcpyAsync(d_cum.p, hc.data(), 4 * hc.size(), cudaMemcpyHostToDevice, st))
        return EP_ECUDA;
    ra.freq = d_freq.as<uint32_t>();
    ra.cum = d_cum.as<uint32_t>();
    k_rans<<<grid_for(T * 32, 128), 128, 0, st>>>(d_fields.as<int32_t>(), nvec, V, T, b, ra,
                                                  d_scratch.as<uint16_t>(), d_nwords.as<uint32_t>(),
                                                  r.states.as<uint32_t>());
    std::vector<uint32_t> nw((size_t)T), off((size_t)T);
    if (cudaMemcpyAsync(nw.data(), d_nwords.p, 4 * T, cudaMemcpyDeviceToHost, st) || cudaStreamSynchronize(st))
        return EP_ECUDA;
    uint64_t words = 0;
    for (int64_t t = 0; t < T; ++t) {
        if (words >= 0xFFFFFFFFull) return EP_EINVAL;
        off[t] = (uint32_t)words;
        words += nw[t];
    }
    if (words > 0xFFFFFFFFull) return EP_EINVAL;
    if (r.payload.alloc(sizeof(uint16_t) * std::max<uint64_t>(words, 1), st) ||
        cudaMemcpyAsync(r.off.p, off.data(), 4 * T, cudaMemcpyHostToDevice, st))
        return EP_ECUDA;
    k_copy_out<<<(unsigned)T, 256, 0, st>>>(d_scratch.as<uint16_t>(), V, d_nwords.as<uint32_t>(), r.off.as<uint32_t>(),
                                            r.payload.as<uint16_t>());
    r.words = words;
    r.b = b;
    r.s = s;
    return cudaGetLastError() == cudaSuccess ? EP_OK : EP_ECUDA;  // the callers synchronise
}

}  // namespace
}  // namespace ep

extern "C" ep_status ep_encode_tensor_gpu(void* stream, const float* W, int64_t rows, int64_t cols,
                                          double target_bpp, const ep_encode_opts* opts, ep_blob** out) {
    using namespace ep;
    if (!W || !out) return EP_EINVAL;
    *out = nullptr;
    if ((reinterpret_cast<uintptr_t>(W) & 3u) != 0) return EP_EINVAL;
    ep_encode_opts o{};
    if (opts) o = *opts;
    int64_t V = 0, T = 0;
    ep_status as = check_encode_args(W, rows, cols, target_bpp, o, V, T);
    if (as != EP_OK) return as;
    try {
        int dev = 0, nsm = 0;
        if ((as = device_for(W, dev, nsm)) != EP_OK) return as;
        const cudaStream_t st = static_cast<cudaStream_t>(stream);
        Encoded r;
        if ((as = encode_core(st, nsm, W, rows, cols, target_bpp, o, V, T, r)) != EP_OK) return as;
        ep_blob* bl = host::new_blob(rows, cols, r.b, V, T, r.words, r.tabs);
        if (!bl) return EP_ENOMEM;
        std::vector<uint32_t> states((size_t)kLanes * T), offs((size_t)T);
        cudaError_t e = cudaMemcpyAsync(bl->payload, r.payload.p, 2 * r.words, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(states.data(), r.states.p, 4 * states.size(), cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(offs.data(), r.off.p, 4 * T, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(bl->row_scales, r.scales.p, sizeof(float) * rows, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) {
            ep_free_blob(bl);
            return EP_ECUDA;
        }
        for (int64_t t = 0; t < T; ++t) {
            bl->tile_index[kTileWords * t] = offs[t];
            for (int j = 0; j < kLanes; ++j) bl->tile_index[kTileWords * t + 1 + j] = states[(size_t)kLanes * t + j];
        }
        bl->tile_index[kTileWords * T] = (uint32_t)r.words;
        host::finish_blob(bl, r.s, o.has_container_scales != 0);
        *out = bl;
        return EP_OK;
    } catch (const std::bad_alloc&) {
        return EP_ENOMEM;
    }
}

extern "C" ep_status ep_encode_tensor_gpu_device(void* stream, const void* W, int w_is_bf16, int64_t rows,
                                                 int64_t cols, double target_bpp, const ep_encode_opts* opts,
                                                 ep_device_blob* out) {
    using namespace ep;
    if (!W || !out) return EP_EINVAL;
    *out = ep_device_blob{};
    if ((reinterpret_cast<uintptr_t>(W) & (w_is_bf16 ? 1u : 3u)) != 0) return EP_EINVAL;
    ep_encode_opts o{};
    if (opts) o = *opts;
    int64_t V = 0, T = 0;
    ep_status as = check_encode_args(W, rows, cols, target_bpp, o, V, T);
    if (as != EP_OK) return as;
    try {
        int dev = 0, nsm = 0;
        if ((as = device_for(W, dev, nsm)) != EP_OK) return as;
        const cudaStream_t st = static_cast<cudaStream_t>(stream);
        DevBuf wide;
        const float* W32 = static_cast<const float*>(W);
        if (w_is_bf16) {
            const int64_t n = rows * cols;
            if (wide.alloc(sizeof(float) * (size_t)n, st) != cudaSuccess) return EP_ECUDA;
            k_widen_bf16<<<std::min(grid_for(n, 256), 16 * nsm), 256, 0, st>>>(static_cast<const uint16_t*>(W), n,
                                                                              wide.as<float>());
            W32 = wide.as<float>();
        }
        Encoded r;
        if ((as = encode_core(st, nsm, W32, rows, cols, target_bpp, o, V, T, r)) != EP_OK) return as;
        // the stream's own buffers, outliving the call
        ep_device_blob d = {};
        d.rows = rows;
        d.cols = cols;
        d.b = r.b;
        d.V = (int)V;
        d.ntiles = (int)T;
        d.payload_words = r.words;
        d.payload_alloc_words = (r.words + 7) / 8 * 8;
        const size_t alloc_words = std::max<size_t>(d.payload_alloc_words, 8);
        d.freq_bytes = host::table_bytes(r.tabs);
        std::vector<uint8_t> ft(d.freq_bytes, 0);
        host::write_tables(ft.data(), rows, cols, r.b, V, T, r.tabs);
        void *pp = nullptr, *pt = nullptr, *pf = nullptr, *ps = nullptr;
        cudaError_t e = cudaMalloc(&pp, 2 * alloc_words);
        if (e == cudaSuccess) e = cudaMalloc(&pt, 4 * ((size_t)kTileWords * T + 1));
        if (e == cudaSuccess) e = cudaMalloc(&pf, d.freq_bytes);
        if (e == cudaSuccess) e = cudaMalloc(&ps, sizeof(float) * rows);
        d.payload = static_cast<uint16_t*>(pp);
        d.tile_index = static_cast<uint32_t*>(pt);
        d.freq_tables = static_cast<uint8_t*>(pf);
        d.row_scales = static_cast<float*>(ps);
        if (e == cudaSuccess) e = cudaMemcpyAsync(pp, r.payload.p, 2 * r.words, cudaMemcpyDeviceToDevice, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(d.payload + r.words, 0, 2 * (alloc_words - r.words), st);
        if (e == cudaSuccess) {
            k_tile_index<<<grid_for(kTileWords * T + 1, 256), 256, 0, st>>>(T, r.off.as<uint32_t>(),
                                                                            r.states.as<uint32_t>(),
                                                                            (uint32_t)r.words, d.tile_index);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) e = cudaMemcpyAsync(pf, ft.data(), d.freq_bytes, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(ps, r.scales.p, sizeof(float) * rows, cudaMemcpyDeviceToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);  // ft (host) is freed on return
        if (e != cudaSuccess) {
            ep_free_device_blob(&d);
            return EP_ECUDA;
        }
        d.s = r.s;
        d.stored_bytes = host::stored_bytes(r.words, T, d.freq_bytes, rows, o.has_container_scales != 0);
        d.stored_bpp = 8.0 * (double)d.stored_bytes / (double)(rows * cols);
        *out = d;
        return EP_OK;
    } catch (const std::bad_alloc&) {
        return EP_ENOMEM;
    }
}

extern "C" void ep_free_device_blob(ep_device_blob* d) {
    if (!d) return;
    if (d->payload) cudaFree(d->payload);
    if (d->tile_index) cudaFree(d->tile_index);
    if (d->freq_tables) cudaFree(d->freq_tables);
    if (d->row_scales) cudaFree(d->row_scales);
    *d = ep_device_blob{};
}
