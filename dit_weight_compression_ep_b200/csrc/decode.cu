// decode.cu -- fused EntroPack weight reconstruction for B200 (sm_100a).
//
// EntroPack paper, Fig. 2b: the GPU decode runs the rANS symbol decode, the
// lattice point, the per-row scale and the output conversion in one pass; §3.6:
// a warp per tile, a lane per interleaved state; App. C.3 tile layout, state
// normalisation and the decoder's lookup tables (shared memory, or a packed
// global form when they do not fit).
//
// One call = one cooperative launch of decode_kernel on the caller's stream:
// one persistent CTA of 24 warps per SM (all co-resident).  Its prologue parses
// the header (lane-parallel checks: it runs once, from a cold instruction cache,
// so its length is its cost) and loads, together, the tables' frequencies of
// this CTA's table, the coset table and every warp's first tile record.  Then
// the CTAs sharing a table (G/16 of them) build its part of the decode-LUT image
// in a stream-ordered global workspace (binary search of every slot in the
// table's cumulative frequencies), arrive on a 64-bit grid counter, wait
// (bounded) for every CTA, and copy the whole image into shared memory with
// cp.async.bulk.  Three image formats (16 coordinate tables, table 2(k-1) + c):
//   PACKED (b <= 11, z fits): a 32-bit entry per slot, low to high
//     [f : b+1][z + even bias][slot - cum : b], or [f - 1 : b][z][slot - cum : b]
//     when z needs the extra bit;
//   TWO (b <= 12 otherwise, the alphabets small enough): a u16 symbol index per
//     slot (per slot pair at b = 12, the odd slot's offset in 4 bits) and the
//     tables' u16 cumulative counts: f = cum[s+1] - cum[s], z = s + min;
//   COARSE (otherwise): a 64-bit entry per bucket of 2^(b-k) slots (k <= 10)
//     {cum | f << 16, z} of the symbol owning the bucket's first slot, and a
//     bounded walk over the global frequencies.
// Tile t goes to CTA t mod G and, within the CTA, to warp (t / G) mod 24.
// Per warp and tile:
//   a1  32 terminal states (one per lane), the tile's payload offsets;
//   a3  payload words staged by cp.async.bulk into a double-buffered ring of
//       2 x 512 words; a chunk landing in the first half is also copied to a
//       288-word mirror after the ring so that one round (at most 288 words)
//       reads without wrapping;
//   a4  per round r each lane decodes the 9 fields (c, z1..z7, m) of vector
//       32r + lane; the coset bit needs no LUT (two symbols, one compare); the
//       lanes that renormalise read consecutive words in ascending lane order
//       (ballot + popc);
//   a5  z8 = 2m + parity(z1..z7), y = z + c/2;
//   a6  w = fl32(sigma_row * y): y = z + c/2 is formed exactly in FP32 (from the
//       bits of 1.5*2^22 + (2z + c)/2) and multiplied once by sigma, so every
//       weight gets a single rounding, whatever sigma;
//   a7  cvt.rn bf16x2 / f16x2, cvt.rn.satfinite e4m3x2, or rni + clamp for
//       INT8 (and + 128 for UINT8), and one 16-byte (8-byte) store per lane, so a warp writes 512
//       (256) contiguous bytes per round.
// The integer arithmetic of a symbol step is split between the logic/shift
// unit and integer multiply-adds (run-time multipliers, on the FMA pipe), and
// each coordinate is formed as soon as its field is decoded.
// Stream errors never fault or trap: every shared-memory index is masked or
// bounded, every global read stays inside the buffers the header describes,
// every wait is bounded, and inconsistencies raise bits in a device status word.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <new>
#include <vector>
#include <type_traits>

#include "entropack.h"
#include "ep_format.h"

namespace ep {
namespace {

constexpr int kWarps = 24;
constexpr int kThreads = 32 * kWarps;
constexpr int kChunkWords = 512;               // words per staged chunk
constexpr int kChunkShift = 9;
constexpr int kRingWords = 2 * kChunkWords;    // double buffer
constexpr int kRoundWords = kFields * kLanes;  // 288: most words one round can consume
constexpr int kRingAllocBytes = 2688;          // (1024 + 288) words, rounded up to 128 bytes
constexpr int kCoarseBits = 10;                // COARSE: at most 2^10 buckets per table

// decode_kernel shared-memory layout (bytes)
constexpr int kLutBytes = 128 * 1024;
constexpr int kOffLut = 0;
constexpr int kOffRing = kOffLut + kLutBytes;
constexpr int kOffBar = kOffRing + kWarps * kRingAllocBytes;  // 2 per warp + 1 for the LUT
constexpr int kOffDesc = kOffBar + kWarps * 16 + 16;
constexpr int kOffDesc2 = kOffDesc + 3 * 32 * 4;  // TWO: per table {record address, min}
constexpr int kSmemBytes = kOffDesc2 + 16 * 8;
// TWO: slot table in the first 64 KiB of the LUT region, cumulative-count records after it
constexpr int kTwoRec = 64 * 1024;
constexpr uint32_t kTwoRecMax = 32 * 1024;  // u16 records: sum over tables 1..16 of (A + 1), + 1

// LUT workspace (global, one per device, zeroed once): the image, then the
// grid barrier's 64-bit arrival counter, which only grows (by G per launch)
constexpr int kWsCountOffset = kLutBytes;
constexpr int kWsBytes = kLutBytes + 32;
constexpr uint32_t kGridSpins = 1u << 22;  // bound on the grid-barrier polls
// A prepared table (ep_decode_prepare): the image, then a trailer at kLutBytes of
// {magic, bad tables, fingerprint lo, fingerprint hi, image bytes}; same size as the workspace.
constexpr uint32_t kLutMagic = 0x5450454Cu;
static_assert(kWsBytes == EP_LUT_BYTES, "prepared table size");
// ep_decode_prepare's kernel: the scan scratch (A + 1 <= 2^15 + 1 u16), then the descriptors
constexpr int kPrepOffDesc = 65536 + 128;
constexpr int kPrepSmemBytes = kPrepOffDesc + 3 * 32 * 4;

// status bits
constexpr unsigned kStCorrupt = 1u;      // payload / state / offset inconsistent
constexpr unsigned kStHeader = 2u;       // table header or tables invalid
constexpr unsigned kStUnsupported = 4u;  // a format variant this decoder does not handle
constexpr unsigned kStTimeout = 8u;      // a bulk copy did not complete in time

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr uint32_t kWaitSpins = 1u << 20;  // bound on mbarrier polls

// Output modes of ep_decode_gemv (not ep_dtype values): the decoded FP32 weights multiplied
// by NT rows of activations inside the decode, NT = mode - kGemv.
constexpr int kGemv = 100;
template <int DT>
__host__ __device__ constexpr int gemv_tokens() { return DT > kGemv ? DT - kGemv : 0; }

// PACKED modes: b (entries hold f - 1) or 16 + b (entries hold f; one add fewer
// per symbol, needs one more bit); COARSE otherwise.
enum : int { kModeCoarse = 1, kModeTwo = 2, kModeTwoPair = 3, kModeF = 16 };

}  // namespace

__device__ unsigned int g_decode_status;

namespace {

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait; returns false when the bound ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t spins = 0; spins < kWaitSpins; ++spins)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
__device__ __forceinline__ void fence_proxy_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ unsigned long long ld_acquire_gpu(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}
__device__ __forceinline__ void raise_status(unsigned bits) { atomicOr(&g_decode_status, bits); }
// Shared-memory loads at 32-bit shared addresses.  The "memory" clobber keeps
// them after the barrier waits that publish the data they read.
template <int OFF = 0>
__device__ __forceinline__ uint32_t ld_s32(uint32_t a) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF) : "memory");
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint2 ld_s64(uint32_t a) {
    uint2 v;
    asm("ld.shared.v2.u32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_s16(uint32_t a) {
    uint32_t v;
    asm("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}

// ------------------------------------------------------------ header checks

struct Geo {
    uint32_t b, V, T, M;
    int mode;
    uint32_t k;            // COARSE: log2 buckets per table
    uint32_t image_bytes;  // bytes of the LUT image
    int64_t nvec;
};

// Parse and check the table header.  Every warp reads the same words and takes
// the same decisions, so the result is uniform; lane t (t < 17) also returns
// table t's {min, A}.  The checks are lane-parallel and division-free: this
// code runs once per CTA, cold, so its length is what it costs.  Returns 0,
// kStHeader or kStUnsupported.
__device__ unsigned parse_header(const uint8_t* ft, int64_t rows, int64_t cols, Geo& g, int& mn, uint32_t& A) {
    const int lane = threadIdx.x & 31;
    uint32_t h[12];
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(ft) + i);
        h[4 * i] = v.x;
        h[4 * i + 1] = v.y;
        h[4 * i + 2] = v.z;
        h[4 * i + 3] = v.w;
    }
    mn = 0;
    A = 0;
    if (lane < kTables) {
        const uint2 d = __ldg(reinterpret_cast<const uint2*>(ft + kHeaderFixedBytes) + lane);
        mn = static_cast<int>(d.x);
        A = d.y;
    }
    g.b = h[kHB];
    g.V = h[kHV];
    g.T = h[kHT];
    g.nvec = rows * ((cols + 7) / 8);  // rows padded to whole vectors
    const int64_t hrows = (int64_t)(((uint64_t)h[2 * kHRows64 + 1] << 32) | h[2 * kHRows64]);
    const int64_t hcols = (int64_t)(((uint64_t)h[2 * kHCols64 + 1] << 32) | h[2 * kHCols64]);
    bool ok = h[kHMagic] == kMagic && h[kHVersion] == kVersion && h[kHJ] == (uint32_t)kLanes &&
              g.b >= (uint32_t)kMinB && g.b <= (uint32_t)kMaxB && g.V >= 1 && g.T >= 1 && hrows == rows &&
              hcols == cols;
    // T = ceil(nvec / V): (T - 1) V < nvec <= T V
    ok = ok && (uint64_t)g.T * g.V >= (uint64_t)g.nvec && (uint64_t)(g.T - 1) * g.V < (uint64_t)g.nvec;
    if (!ok) return kStHeader;
    if (h[kHNTab] != (uint32_t)kTables || h[kHFlags] != 0u) return kStUnsupported;
    g.M = 1u << g.b;
    // per table (one lane each): alphabet within 2^b, the coset table {0, 1}-valued; whether
    // z fits the packed entry with (fstored) and without the extra f bit
    const int bb = g.b <= 11 ? (int)g.b : 11;
    const int64_t zlim = 1ll << (31 - 2 * bb), zlim_f = 1ll << (30 - 2 * bb);
    bool badt = A > g.M;
    if (lane == 0) badt |= A < 1 || A > 2 || mn < 0 || mn + (int)A > 2;
    const bool coord = lane >= 1 && lane < kTables && A > 0;
    const int64_t zhi = (int64_t)mn + A - 1;
    const bool pk = !coord || (mn >= -zlim && zhi < zlim);
    const bool fs = !coord || (mn >= -zlim_f && zhi < zlim_f);
    if (__any_sync(kFull, badt)) return kStHeader;
    const bool packed = g.b <= 11 && __all_sync(kFull, pk);
    const bool fstored = g.b <= 11 && __all_sync(kFull, fs);
    // TWO: records of tables 1..16 (A + 1 each) and one pad entry
    const uint32_t nrec = 1u + __reduce_add_sync(kFull, lane >= 1 && lane < kTables ? A + 1u : 0u);
    const bool two = g.b <= 12 && nrec <= kTwoRecMax;
    g.mode = fstored ? kModeF + (int)g.b
                     : (packed ? (int)g.b : (two ? (g.b == 12 ? kModeTwoPair : kModeTwo) : kModeCoarse));
    g.k = g.b < (uint32_t)kCoarseBits ? g.b : (uint32_t)kCoarseBits;
    if (g.mode == kModeTwo || g.mode == kModeTwoPair)
        g.image_bytes = (uint32_t)kTwoRec + ((2u * nrec + 15u) & ~15u);
    else
        g.image_bytes = packed ? 16u * g.M * 4u : 16u * (1u << g.k) * 8u;
    return 0;
}

// A fingerprint of what fixes the LUT image's layout: b, the LUT format and every table's
// {min, A}.  Warp-uniform; a SplitMix64 finaliser per lane, summed in two 32-bit halves.
__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}
__device__ __forceinline__ uint2 table_fingerprint(const Geo& g, int mn, uint32_t A) {
    const int lane = threadIdx.x & 31;
    uint64_t v = 0;
    if (lane < kTables) v = mix64(((uint64_t)lane << 56) ^ ((uint64_t)(uint32_t)mn << 20) ^ (uint64_t)A);
    else if (lane == 31) v = mix64((0xE8ull << 56) ^ ((uint64_t)g.b << 8) ^ (uint64_t)(uint32_t)g.mode);
    return make_uint2(__reduce_add_sync(kFull, (uint32_t)v), __reduce_add_sync(kFull, (uint32_t)(v >> 32)));
}

// ------------------------------------------------------- LUT image slice

// a2, part 1.  Every CTA builds 1/G of the decode-LUT image in the global
// workspace: 16 tables x E entries (E = 2^b slots for PACKED, 2^k buckets for
// COARSE); its range touches at most two tables.  For each touched table the
// CTA scans the frequencies into cumulative counts (u16; M <= 2^15) in shared
// scratch and finds the owner of every slot by binary search.  Returns true
// when a touched table does not sum to 2^b.
constexpr int kPre = 6;  // a table of up to kPre * kThreads symbols comes in with the prologue's loads

__device__ __forceinline__ bool build_lut_slice(const Geo& g, const uint16_t* fq, const int* s_min,
                                                const uint32_t* s_A, const uint32_t* s_off, uint8_t* ws,
                                                uint16_t* scratch, int t_pre, const uint32_t (&fr)[kPre]) {
    __shared__ uint32_t part_sum[kWarps];
    const bool coarse = g.mode == kModeCoarse;
    const bool fstored = g.mode >= kModeF;
    const bool two = g.mode == kModeTwo || g.mode == kModeTwoPair, pair = g.mode == kModeTwoPair;
    const uint32_t E = coarse ? (1u << g.k) : (pair ? g.M / 2u : g.M);
    const uint32_t sh = coarse ? g.b - g.k : 0u;
    uint32_t e0, e1;
    if (gridDim.x >= 16) {
        // CTAs [ceil(tG/16), ceil((t+1)G/16)) share table t + 1, so no CTA builds two tables
        const uint32_t G = gridDim.x, t0 = blockIdx.x * 16u / G;
        const uint32_t bf = (t0 * G + 15u) / 16u, n = ((t0 + 1u) * G + 15u) / 16u - bf, j = blockIdx.x - bf;
        e0 = t0 * E + j * E / n;  // j < n <= G, E <= 2^15
        e1 = t0 * E + (j + 1u) * E / n;
    } else {
        const uint32_t all = 16u * E;
        const uint32_t per = (all + gridDim.x - 1) / gridDim.x;
        e0 = min(all, blockIdx.x * per);
        e1 = min(all, e0 + per);
    }
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    bool bad = false;
    if (e0 >= e1) return false;
    const int tfirst = 1 + (int)(e0 / E), tlast = 1 + (int)((e1 - 1) / E);
    for (int t = tfirst; t <= tlast; ++t) {
        uint16_t* cum = scratch;  // one table at a time: A + 1 <= 2^15 + 1 entries
        const uint32_t A = s_A[t], off = s_off[t];
        const int mn = s_min[t];
        // frequencies into shared memory, then an in-place exclusive scan by contiguous chunks
        if (t == t_pre) {  // frequencies already in registers
#pragma unroll
            for (int k = 0; k < kPre; ++k) {
                const uint32_t q = (uint32_t)tid + (uint32_t)k * kThreads;
                if (q < A) cum[q] = (uint16_t)fr[k];
            }
        } else {
            for (uint32_t q = tid; q < A; q += kThreads) cum[q] = fq[off + q];
        }
        __syncthreads();
        const uint32_t chunk = (A + kThreads - 1) / kThreads;
        const uint32_t q0 = min(A, tid * chunk), q1 = min(A, q0 + chunk);
        uint32_t local = 0;
        for (uint32_t q = q0; q < q1; ++q) local += cum[q];
        uint32_t incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) part_sum[wid] = incl;
        __syncthreads();
        const uint32_t ps = lane < kWarps ? part_sum[lane] : 0u;
        const uint32_t before = __reduce_add_sync(kFull, lane < wid ? ps : 0u);
        const uint32_t total = __reduce_add_sync(kFull, ps);
        uint32_t run = before + incl - local;
        for (uint32_t q = q0; q < q1; ++q) {
            const uint32_t f = cum[q];
            cum[q] = (uint16_t)(run < g.M ? run : g.M);
            run += f;
        }
        if (tid == 0) cum[A] = (uint16_t)(total < g.M ? total : g.M);
        __syncthreads();
        const bool valid = A == 0 || total == g.M;
        bad |= !valid;
        // entries of this table inside [e0, e1)
        const uint32_t lo = max(e0, (uint32_t)(t - 1) * E), hi = min(e1, (uint32_t)t * E);
        if (two && lo == (uint32_t)(t - 1) * E) {
            // the CTA holding the table's first entry writes its records: cum_0 .. cum_{A-1}, M
            // (tables 1..16 back to back, A + 1 records each)
            uint16_t* rec = reinterpret_cast<uint16_t*>(ws + kTwoRec) + (s_off[t] - s_A[0] + (uint32_t)(t - 1));
            for (uint32_t q = tid; q <= A; q += kThreads) rec[q] = q < A ? cum[q] : (uint16_t)g.M;
            if (t == 16 && tid == 0) rec[A + 1] = (uint16_t)g.M;  // pad: a zero entry of the last table reads it
        }
        if (two) {
            for (uint32_t idx = lo + tid; idx < hi; idx += kThreads) {
                const uint32_t j = idx - (uint32_t)(t - 1) * E;
                uint32_t e = 0;
                if (A > 0 && valid) {
                    // the largest s with cum[s] <= slot owns the slot (zero-frequency symbols
                    // share their successor's count and are passed over)
                    const uint32_t slot = pair ? 2u * j : j;
                    uint32_t l = 0, r = A;
                    while (r - l > 1) {
                        const uint32_t mid = (l + r) >> 1;
                        if (cum[mid] <= slot) l = mid;
                        else r = mid;
                    }
                    e = l;
                    if (pair) {  // the odd slot's owner, as an offset of at most 15 (15: look further)
                        uint32_t so = l;
                        while (so + 1 < A && so < l + 15u && cum[so + 1] <= slot + 1u) ++so;
                        e |= (so - l) << 12;
                    }
                }
                reinterpret_cast<uint16_t*>(ws)[idx] = (uint16_t)e;
            }
            __syncthreads();  // the scratch is reused by the next table
            continue;
        }
        for (uint32_t idx = lo + tid; idx < hi; idx += kThreads) {
            const uint32_t j = idx - (uint32_t)(t - 1) * E;  // slot (PACKED) or bucket (COARSE)
            const uint32_t slot = j << sh;
            uint32_t s = 0, c0 = 0, f = 0;
            if (A > 0 && valid) {
                uint32_t l = 0, r = A;  // cum[l] <= slot < cum[r]
                while (r - l > 1) {
                    const uint32_t mid = (l + r) >> 1;
                    if (cum[mid] <= slot) l = mid;
                    else r = mid;
                }
                s = l;
                c0 = cum[s];
                f = cum[s + 1] - c0;
            }
            if (coarse) {
                reinterpret_cast<uint2*>(ws)[idx] =
                    A > 0 && valid ? make_uint2(c0 | (f << 16), (uint32_t)((int)s + mn)) : make_uint2(0u, 0u);
            } else {
                const uint32_t b = g.b;
                uint32_t e = 0;
                if (A > 0 && valid)
                    e = fstored ? f | ((uint32_t)((int)s + mn + (1 << (30 - 2 * b))) << (b + 1)) | ((slot - c0) << (32 - b))
                                : (f - 1) | ((uint32_t)((int)s + mn + (1 << (31 - 2 * b))) << b) | ((slot - c0) << (32 - b));
                reinterpret_cast<uint32_t*>(ws)[idx] = e;
            }
        }
        __syncthreads();  // the scratch is reused by the next table
    }
    return bad;
}

// ------------------------------------------------------------ output writers

template <int DT>
struct Out;

// One element of the output type (the element-wise path of rows padded to whole vectors).
template <int DT>
__device__ __forceinline__ void put_elem(void* out, int64_t i, float w) {
    if constexpr (DT == EP_BF16) {
        reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(w);
    } else if constexpr (DT == EP_FP16) {
        reinterpret_cast<__half*>(out)[i] = __float2half_rn(w);
    } else if constexpr (DT == EP_FP8_E4M3) {
        reinterpret_cast<__nv_fp8_storage_t*>(out)[i] = __nv_cvt_float_to_fp8(w, __NV_SATFINITE, __NV_E4M3);
    } else if constexpr (DT == EP_INT8) {
        reinterpret_cast<int8_t*>(out)[i] = (int8_t)__float2int_rn(fminf(fmaxf(w, -127.0f), 127.0f));
    } else if constexpr (DT == EP_UINT8) {
        reinterpret_cast<uint8_t*>(out)[i] = (uint8_t)(__float2int_rn(fminf(fmaxf(w, -128.0f), 127.0f)) + 128);
    } else {
        reinterpret_cast<float*>(out)[i] = w;
    }
}

template <>
struct Out<EP_BF16> {
    __device__ static void store(void* out, int64_t g, const float w[8]) {
        __nv_bfloat162 a = __floats2bfloat162_rn(w[0], w[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(w[2], w[3]);
        __nv_bfloat162 c = __floats2bfloat162_rn(w[4], w[5]);
        __nv_bfloat162 d = __floats2bfloat162_rn(w[6], w[7]);
        uint4 v;
        v.x = *reinterpret_cast<uint32_t*>(&a);
        v.y = *reinterpret_cast<uint32_t*>(&b);
        v.z = *reinterpret_cast<uint32_t*>(&c);
        v.w = *reinterpret_cast<uint32_t*>(&d);
        reinterpret_cast<uint4*>(out)[g] = v;
    }
};
template <>
struct Out<EP_FP16> {
    __device__ static void store(void* out, int64_t g, const float w[8]) {
        __half2 a = __floats2half2_rn(w[0], w[1]);
        __half2 b = __floats2half2_rn(w[2], w[3]);
        __half2 c = __floats2half2_rn(w[4], w[5]);
        __half2 d = __floats2half2_rn(w[6], w[7]);
        uint4 v;
        v.x = *reinterpret_cast<uint32_t*>(&a);
        v.y = *reinterpret_cast<uint32_t*>(&b);
        v.z = *reinterpret_cast<uint32_t*>(&c);
        v.w = *reinterpret_cast<uint32_t*>(&d);
        reinterpret_cast<uint4*>(out)[g] = v;
    }
};
template <>
struct Out<EP_FP8_E4M3> {
    __device__ static void store(void* out, int64_t g, const float w[8]) {
        uint32_t q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            q[i] = __nv_cvt_float2_to_fp8x2(make_float2(w[2 * i], w[2 * i + 1]), __NV_SATFINITE, __NV_E4M3);
        uint2 v;
        v.x = __byte_perm(q[0], q[1], 0x5410);
        v.y = __byte_perm(q[2], q[3], 0x5410);
        reinterpret_cast<uint2*>(out)[g] = v;
    }
};
// INT8 / UINT8: the clamped value plus 1.5 * 2^23 (+ 128 for UINT8) lands in [2^23, 2^24), where
// the float spacing is 1, so the addition rounds to the nearest integer, ties to even, and the
// low byte of the sum's bits is the integer's byte.  This keeps the conversion on the FMA pipe.
__device__ __forceinline__ int round_to_byte(float v, float magic) { return __float_as_int(v + magic); }

template <>
struct Out<EP_INT8> {
    __device__ static void store(void* out, int64_t g, const float w[8]) {
        int q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = round_to_byte(fminf(fmaxf(w[i], -127.0f), 127.0f), 12582912.0f);
        uint2 v;
        v.x = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
        v.y = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
        reinterpret_cast<uint2*>(out)[g] = v;
    }
};
template <>
struct Out<EP_UINT8> {
    __device__ static void store(void* out, int64_t g, const float w[8]) {
        int q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = round_to_byte(fminf(fmaxf(w[i], -128.0f), 127.0f), 12583040.0f);
        uint2 v;
        v.x = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
        v.y = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
        reinterpret_cast<uint2*>(out)[g] = v;
    }
};
template <>
struct Out<EP_FP32> {
    __device__ static void store(void* out, int64_t g, const float w[8]) {
        float4* o = reinterpret_cast<float4*>(out) + 2 * g;
        o[0] = make_float4(w[0], w[1], w[2], w[3]);
        o[1] = make_float4(w[4], w[5], w[6], w[7]);
    }
};

// ------------------------------------------------------------- symbol LUTs

// PACKED: 16 tables x 2^B slots x 32-bit entries at shared address lut_s;
// table (2(k-1) + c).  Entry, low to high: f in B+1 bits (F) or f - 1 in B bits,
// then z with an even bias (31 - 2B or 32 - 2B bits), then slot - cum in the top
// B bits, so that f and slot - cum each come out in one operation.
//
// decode<K> returns the entry shifted right so that bits 1.. hold z + bias (kZMask
// selects them, bit 0 is cleared by the mask): twice the biased coordinate, ready to be
// OR-ed into the float magic of the reconstruction with the coset bit in bit 0.  For the
// last field (m) the shift is one less, so that kZMask << 1 gives four times it.
template <int B, bool F>
struct PackedLut {
    static constexpr uint32_t kM = 1u << B;
    static constexpr int kB = B;
    static constexpr bool kPacked = true;
    static constexpr uint32_t kZBias = F ? (1u << (30 - 2 * B)) : (1u << (31 - 2 * B));
    static constexpr int kZShift = F ? B : B - 1;  // entry bit of z's lowest bit, minus one
    static constexpr uint32_t kZMask = ((1u << (F ? 31 - 2 * B : 32 - 2 * B)) - 1u) << 1;
    uint32_t lut_s;
    uint32_t four;  // 4 and 2^32 - 4 * 2^B: run-time values, so that the address
    uint32_t m4;    // arithmetic stays integer multiply-adds
    __device__ __forceinline__ uint32_t coset_base(int c) const { return lut_s + ((uint32_t)c << (B + 2)); }
    template <int K>
    __device__ __forceinline__ uint32_t decode(uint32_t& x, uint32_t cb, bool& bad) const {
        const uint32_t xs = x >> B;
        const uint32_t a = xs * m4 + (x * four + cb);  // cb + 4 (x mod 2^B)
        const uint32_t e = ld_s32<(2 * (K - 1)) * (int)kM * 4>(a);
        const uint32_t f = e & (F ? 2u * kM - 1u : kM - 1u);
        const uint32_t bias = e >> (32 - B);
        if constexpr (F) {
            x = f * xs + bias;
        } else {
            x = f * xs + (xs + bias);
        }
        (void)bad;
        return K < 8 ? e >> kZShift : e >> (kZShift - 1);
    }
};

// TWO: a u16 per slot (b <= 11) or per slot pair (b = 12, PAIR) holding the table-local
// symbol index s (and, for a pair, the odd slot's offset from it, 15 meaning "at least
// 15"), then the table's u16 cumulative counts cum[s], cum[s + 1]: f = cum[s + 1] - cum[s],
// slot - cum[s], z = s + min.  Runtime b.
template <bool PAIR>
struct TwoLut {
    static constexpr int kB = 0;
    static constexpr bool kPacked = false;
    static constexpr bool kYbDirect = true;
    static constexpr uint32_t kZBias = 0;
    uint32_t lut_s;  // slot table (tables in the order 2(k-1) + c)
    uint32_t b, mmask, half;  // b, 2^b - 1, 2 * entries per table (bytes per table)
    uint32_t desc_s;          // shared address of {record address, 0x4AC00000 + c + 2 min (4 min for m)}
    const uint32_t* s_A;      // alphabet sizes, for the escape walk
    __device__ __forceinline__ uint32_t coset_base(int c) const { return (uint32_t)c; }
    template <int K>
    __device__ __forceinline__ uint32_t decode(uint32_t& x, uint32_t c, bool& bad) const {
        const uint32_t tix = 2u * (K - 1) + c;  // table t - 1
        const uint2 d = ld_s64<8 * 2 * (K - 1)>(desc_s + 8u * c);
        const uint32_t slot = x & mmask;
        const uint32_t xs = x >> b;
        uint32_t s;
        if constexpr (PAIR) {
            const uint32_t e = ld_s16(lut_s + tix * half + (x & (mmask - 1u)));
            const uint32_t odd = x & 1u;
            const uint32_t dl = e >> 12;
            s = odd * dl + (e & 4095u);
            if (odd && dl == 15u) {  // a run of unused symbols: walk on (bounded by the alphabet)
                const uint32_t A = s_A[1 + tix];
                while (s + 1u < A && ld_s16(d.x + 2u * (s + 1u)) <= slot) ++s;
            }
        } else {
            s = ld_s16(lut_s + tix * half + 2u * slot);
        }
        const uint32_t ra = d.x + 2u * s;
        const uint32_t c0 = ld_s16(ra), c1 = ld_s16(ra + 2u);
        x = (c1 - c0) * xs + (slot - c0);
        (void)bad;
        // the coordinate's bits: 0x4AC00000 + 2z + c (fields 1..7), 0x4AC00000 + 4m + c (m)
        return s * (K < 8 ? 2u : 4u) + d.y;
    }
};

// COARSE: 16 tables x 2^k buckets x 64-bit {cum | f << 16, z}; runtime b.
struct CoarseLut {
    static constexpr int kB = 0;
    static constexpr bool kPacked = false;
    static constexpr bool kYbDirect = false;
    static constexpr uint32_t kZBias = 0;
    uint32_t lut_s;  // shared address
    uint32_t b, mmask, sh, nb_shift;
    const uint16_t* fq;  // global frequencies
    const int* s_min;
    const uint32_t* s_A;
    const uint32_t* s_off;
    __device__ __forceinline__ uint32_t coset_base(int c) const { return lut_s + ((uint32_t)c << (nb_shift + 3)); }
    template <int K>
    __device__ __forceinline__ uint32_t decode(uint32_t& x, uint32_t cb, bool& bad) const {
        const uint32_t slot = x & mmask;
        const uint2 e = ld_s64(cb + ((uint32_t)(2 * (K - 1)) << (nb_shift + 3)) + ((slot >> sh) << 3));
        uint32_t c0 = e.x & 0xFFFFu, f = e.x >> 16;
        int z = static_cast<int>(e.y);
        if (slot >= c0 + f) {
            const int t = 1 + 2 * (K - 1) + (int)((cb - lut_s) >> (nb_shift + 3));
            const int mn = s_min[t];
            const uint32_t A = s_A[t], off = s_off[t];
            // the walk may cross zero-frequency symbols (unobserved values inside the
            // alphabet), so it is bounded by the alphabet, not by the bucket width
            while (slot >= c0 + f) {
                c0 += f;
                ++z;
                const uint32_t s = (uint32_t)(z - mn);
                if (s >= A) {
                    bad = true;
                    f = 1u;
                    c0 = slot;
                    break;
                }
                f = fq[off + s];
            }
        }
        x = f * (x >> b) + (slot - c0);
        return (uint32_t)z;
    }
};

// ------------------------------------------------------ per-warp payload ring

struct Ring {
    uint8_t* ring;    // this warp's ring (generic pointer into shared memory)
    uint32_t ring_s;  // its shared address
    uint32_t bar_s;   // shared address of its two mbarriers
    uint32_t seq;     // chunks issued so far (all tiles)
    uint32_t waited;  // chunks waited for so far
    bool timed_out;
};

// Issue the next chunk: words [src, src + n) into ring half seq & 1 (and its
// first 288 words to the mirror when that half is the first one).
__device__ __forceinline__ void ring_issue(Ring& rg, const uint16_t* src, uint32_t n, int lane) {
    const uint32_t half = rg.seq & 1u;
    const uint32_t bar = rg.bar_s + 8u * half;
    const uint32_t mirror = half == 0 ? (n < (uint32_t)kRoundWords ? n : (uint32_t)kRoundWords) : 0u;
    if (lane == 0) {
        mbar_arrive_expect_tx(bar, 2u * (n + mirror));
        bulk_g2s(rg.ring_s + 2u * kChunkWords * half, src, 2u * n, bar);
        if (mirror) bulk_g2s(rg.ring_s + 2u * kRingWords, src, 2u * mirror, bar);
    }
    rg.seq += 1;
}

__device__ __forceinline__ void ring_wait_one(Ring& rg) {
    const uint32_t s = rg.waited;
    if (!mbar_wait(rg.bar_s + 8u * (s & 1u), (s >> 1) & 1u)) rg.timed_out = true;
    rg.waited = s + 1;
}

// ------------------------------------------------------------ the decode loop

struct TileCtx {
    int64_t nvec;
    uint32_t V, T, nq, total;
    uint32_t f0c, f1c, cmin;  // coset table: f of symbol 0, of symbol 1, its min
    uint32_t b;
    // 2, 4, 2^16, -2^b, f1c - f0c, -f0c: run-time multipliers (integer multiply-adds run
    // beside the shift / logic / compare unit instead of on it)
    uint32_t two, four, k64, mneg, df, nf0;
    int64_t cols;  // (a width that is not a multiple of 8 pads each row to whole vectors)
    uint32_t cta, G;  // this CTA's rank among the G CTAs that share the tensor: its tiles are cta + i G
    const uint16_t* gx;  // ep_decode_gemv: BF16 activations [tokens, cols]
    float* gy;           // ep_decode_gemv: the product [tokens, rows]
    uint32_t rows;
};

// ep_decode_gemv: a lane's partial dot products for the row its vectors are in.  They go to the
// product when the lane's vectors move on to the next row, and at the tile's end: the lanes that
// leave the same row sum theirs across the warp first, so one atomic add a token carries them.
// The eight BF16 activations of a vector's columns (one 16-byte load a token) come in a round
// ahead for up to 4 tokens, so that their latency hides behind the round's nine symbol steps;
// for 8 tokens they are loaded where they are used (held a round ahead, they would not fit in
// the registers).
template <int NT>
struct GemvAcc {
    static constexpr bool kAhead = NT <= 4;
    float a[NT];
    uint4 xv[kAhead ? NT : 1];
    uint32_t row;  // 0xFFFFFFFF: nothing accumulated
    __device__ __forceinline__ static uint4 xload(const TileCtx& tc, uint32_t q, int t) {
        return __ldg(reinterpret_cast<const uint4*>(tc.gx + (size_t)t * (size_t)tc.cols) + q);
    }
    // the activations of column block q (the lane's vector in the next round)
    __device__ __forceinline__ void ahead(const TileCtx& tc, uint32_t q) {
        if constexpr (kAhead) {
#pragma unroll
            for (int t = 0; t < NT; ++t) xv[t] = xload(tc, q, t);
        }
    }
    // d + x0 w0 + x1 w1 for a pair of BF16 activations and a pair of BF16 weights (low halves
    // first): FP32 multiply-adds of BF16 operands, whose products are exact in FP32
    __device__ __forceinline__ static float fma_pair(uint32_t xp, uint32_t wp, float d) {
        asm("{\n\t.reg .b16 x0, x1, w0, w1;\n\t"
            "mov.b32 {x0, x1}, %1;\n\t"
            "mov.b32 {w0, w1}, %2;\n\t"
            "fma.rn.f32.bf16 %0, x0, w0, %0;\n\t"
            "fma.rn.f32.bf16 %0, x1, w1, %0;\n\t}"
            : "+f"(d)
            : "r"(xp), "r"(wp));
        return d;
    }
    // a[t] += <w, x_t> over the vector's eight columns (block q), w the weights rounded to BF16
    // (the values the BF16 output holds); the activations stay packed
    __device__ __forceinline__ void madd(const TileCtx& tc, uint32_t q, const float* w) {
        uint32_t wb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(w[2 * i], w[2 * i + 1]);
            wb[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            uint4 p;
            if constexpr (kAhead) p = xv[t];
            else p = xload(tc, q, t);
            float d = a[t];
            d = fma_pair(p.x, wb[0], d);
            d = fma_pair(p.y, wb[1], d);
            d = fma_pair(p.z, wb[2], d);
            a[t] = fma_pair(p.w, wb[3], d);
        }
    }
    // the lane's vector of this round is in row r (act: the lane has a vector this round)
    __device__ __forceinline__ void enter(const TileCtx& tc, uint32_t r, bool act) {
        warp_flush(tc, act && row != r && row != 0xFFFFFFFFu);
        if (act) row = r;
    }
    __device__ __forceinline__ void init() {
        row = 0xFFFFFFFFu;
#pragma unroll
        for (int t = 0; t < NT; ++t) a[t] = 0.0f;
    }
    // every lane of the warp calls this; the lanes with `need` add their sums to y and reset them.
    // Lanes that flush the same row add their sums by a butterfly first (one atomic add a token);
    // after two such rows the rest add one by one.
    __device__ __forceinline__ void warp_flush(const TileCtx& tc, bool need) {
        uint32_t bal = __ballot_sync(0xFFFFFFFFu, need);
        for (int pass = 0; pass < 2 && bal; ++pass) {
            const int lead = __ffs(bal) - 1;
            const uint32_t row0 = __shfl_sync(0xFFFFFFFFu, row, lead);
            const bool grp = need && row == row0;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                float v = grp ? a[t] : 0.0f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                if ((int)(threadIdx.x & 31) == lead) atomicAdd(tc.gy + (size_t)t * tc.rows + row0, v);
                if (grp) a[t] = 0.0f;
            }
            if (grp) need = false;
            bal &= ~__ballot_sync(0xFFFFFFFFu, grp);
        }
        if (need) {
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                atomicAdd(tc.gy + (size_t)t * tc.rows + row, a[t]);
                a[t] = 0.0f;
            }
        }
    }
    __device__ __forceinline__ bool pending() const { return row != 0xFFFFFFFFu; }
};
template <>
struct GemvAcc<0> {
    __device__ __forceinline__ void enter(const TileCtx&, uint32_t, bool) {}
    __device__ __forceinline__ void warp_flush(const TileCtx&, bool) {}
    __device__ __forceinline__ void ahead(const TileCtx&, uint32_t) {}
    __device__ __forceinline__ void init() {}
    __device__ __forceinline__ bool pending() const { return false; }
};

// One tile's bookkeeping: record, staging state and every lane's row.
struct Tile {
    uint32_t t;
    int64_t v0;
    uint32_t vt, rounds;
    uint32_t base, fend, nchunks, seq0, org;
    uint32_t off0, off1;
    uint32_t x;
    uint32_t ql, rowl;
    bool ok;
};

__device__ __forceinline__ void tile_issue_chunk(const uint16_t* tiles, Ring& rg, const Tile& tl, uint32_t ci,
                                                 int lane) {
    const uint32_t w0 = tl.base + ci * kChunkWords;
    const uint32_t n = tl.fend - w0 < (uint32_t)kChunkWords ? tl.fend - w0 : (uint32_t)kChunkWords;
    ring_issue(rg, tiles + w0, n, lane);
}

// Read the tile record (loads only: the caller may issue other loads before the
// values are used).
__device__ __forceinline__ void tile_load(const TileCtx& tc, const uint32_t* tix, Tile& tl, uint32_t t, int lane) {
    tl.t = t;
    tl.v0 = (int64_t)t * tc.V;
    tl.vt = (uint32_t)((tc.nvec - tl.v0) < (int64_t)tc.V ? (tc.nvec - tl.v0) : (int64_t)tc.V);
    tl.rounds = (tl.vt + 31) >> 5;
    const uint32_t* rec = tix + (size_t)kTileWords * t;
    tl.off0 = rec[0];
    tl.off1 = rec[kTileWords];
    tl.x = rec[1 + lane];
}

// Check the tile record and start staging its first two chunks.
__device__ __forceinline__ void tile_start(const TileCtx& tc, const uint16_t* tiles, Ring& rg, Tile& tl, int lane) {
    const bool bad = !(tl.off0 <= tl.off1 && tl.off1 <= tc.total) || tl.x < kStateLow || tl.x >= 0x80000000u;
    tl.ok = !__any_sync(kFull, bad);
    tl.base = tl.off0 & ~7u;
    tl.fend = (tl.off1 + 7u) & ~7u;
    tl.nchunks = tl.ok ? (tl.fend - tl.base + kChunkWords - 1) >> kChunkShift : 0u;
    tl.seq0 = rg.seq;
    tl.org = (tl.seq0 & 1u) * kChunkWords;
    if (tl.nchunks > 0) tile_issue_chunk(tiles, rg, tl, 0, lane);
    if (tl.nchunks > 1) tile_issue_chunk(tiles, rg, tl, 1, lane);
    const uint32_t v0 = (uint32_t)tl.v0;  // < nvec < 2^31
    const uint32_t rowbase = v0 / tc.nq;
    tl.ql = v0 - rowbase * tc.nq + lane;
    tl.rowl = rowbase;
    while (tl.ql >= tc.nq) {
        tl.ql -= tc.nq;
        ++tl.rowl;
    }
}

__device__ __forceinline__ void tile_begin(const TileCtx& tc, const uint16_t* tiles, const uint32_t* tix, Ring& rg,
                                           Tile& tl, uint32_t t, int lane) {
    tile_load(tc, tix, tl, t, lane);
    tile_start(tc, tiles, rg, tl, lane);
}

// Renormalisation of every lane after one symbol: the lanes whose state fell
// below 2^15 take the next words in ascending lane order.  pb is the shared
// byte address of the next unread word.
template <bool FULL>
__device__ __forceinline__ void renorm(uint32_t& x, uint32_t xn, bool act, uint32_t& pb, uint32_t lt,
                                       const TileCtx& tc) {
    if constexpr (FULL) {
        // every lane active: one predicate feeds the ballot, the word load and a predicated
        // multiply-add that appends the word (x = xn otherwise)
        asm("{\n\t.reg .pred p;\n\t.reg .b32 bal, t, w;\n\t"
            "setp.lt.u32 p, %2, 32768;\n\t"
            "vote.sync.ballot.b32 bal, p, -1;\n\t"
            "and.b32 t, bal, %3;\n\t"
            "popc.b32 t, t;\n\t"
            "mad.lo.u32 t, t, %4, %1;\n\t"
            "ld.shared.u16 w, [t];\n\t"
            "mov.b32 %0, %2;\n\t"
            "@p mad.lo.u32 %0, %2, %5, w;\n\t"
            "popc.b32 t, bal;\n\t"
            "mad.lo.u32 %1, t, %4, %1;\n\t}"
            : "=r"(x), "+r"(pb)
            : "r"(xn), "r"(lt), "r"(tc.two), "r"(tc.k64)
            : "memory");
        (void)act;
        return;
    }
    const bool need = act && xn < kStateLow;
    const uint32_t bal = __ballot_sync(kFull, need);
    const uint32_t w = ld_s16(__popc(bal & lt) * tc.two + pb);
    const uint32_t xr = xn * tc.k64 + w;  // (xn << 16) | w
    if (act) x = need ? xr : xn;
    pb = __popc(bal) * tc.two + pb;
}

template <int DT, bool RAGGED, typename Lut, bool FULL>
__device__ __forceinline__ void decode_round(void* out, const float sigma, const Lut& lut, const TileCtx& tc,
                                             Tile& tl, uint32_t& pb, uint32_t r, uint32_t lt, int lane,
                                             bool& corrupt, GemvAcc<gemv_tokens<DT>()>& acc, uint32_t q_now) {
    const uint32_t u = (r << 5) + lane;
    const bool act = FULL || u < tl.vt;
    const int64_t g = tl.v0 + u;
    uint32_t x = tl.x;

    // ---- a4: field 0, the coset bit (a two-symbol table: one compare)
    const uint32_t xs = Lut::kB > 0 ? (x >> Lut::kB) : (x >> tc.b);
    const uint32_t slot = xs * tc.mneg + x;
    const uint32_t cs = slot >= tc.f0c ? 1u : 0u;
    {
        const uint32_t f = cs * tc.df + tc.f0c;
        const uint32_t bias = cs * tc.nf0 + slot;
        renorm<FULL>(x, f * xs + bias, act, pb, lt, tc);
    }
    const int c = (int)(tc.cmin + cs);
    const auto cb = lut.coset_base(c & 1);
    bool badsym = false;
    const uint32_t magic = 0x4AC00000u + (uint32_t)c - 2u * Lut::kZBias;
    // packed tables: 0x4AC00000 (1.5 * 2^22) has no bits below bit 22, so the coset bit and
    // twice the biased coordinate are OR-ed in; the bias moves into the float subtraction
    const uint32_t kc = 0x4AC00000u | (uint32_t)c;
    constexpr float kYOff = 6291456.0f + (float)Lut::kZBias;  // exact: below 2^23
    uint32_t yb[8];
    float wf[8];
    uint32_t s7 = 0;
    uint32_t xn;
    // each coordinate's bits as soon as its field is known, so that this work can fill
    // the gaps of the state chain; the parity of z1..z7 is bit 1 of the XOR of the packed
    // tables' shifted entries (the bias is even), or bit 0 of the sum of the others' z
#define EP_FIELD(K)                                               \
    xn = x;                                                       \
    {                                                             \
        const uint32_t z_ = lut.template decode<K>(xn, cb, badsym); \
        renorm<FULL>(x, xn, act, pb, lt, tc);                     \
        if constexpr (Lut::kPacked) {                             \
            if (K < 8) {                                          \
                yb[K - 1] = (z_ & Lut::kZMask) | kc;              \
                wf[K - 1] = sigma * (__uint_as_float(yb[K - 1]) - kYOff); \
                s7 ^= z_;                                         \
            } else {                                              \
                yb[7] = (z_ & (Lut::kZMask << 1)) + (s7 & 2u) + (magic - 2u * Lut::kZBias); \
            }                                                     \
        } else if constexpr (Lut::kYbDirect) {                    \
            if (K < 8) {                                          \
                yb[K - 1] = z_;                                   \
                wf[K - 1] = sigma * (__uint_as_float(yb[K - 1]) - 6291456.0f); \
                s7 ^= z_;                                         \
            } else {                                              \
                yb[7] = z_ + (s7 & 2u);                           \
            }                                                     \
        } else if (K < 8) {                                       \
            yb[K - 1] = z_ * tc.two + magic;                      \
            wf[K - 1] = sigma * (__uint_as_float(yb[K - 1]) - 6291456.0f); \
            s7 += z_;                                             \
        } else {                                                  \
            yb[7] = z_ * tc.four + ((s7 & 1u) * tc.two + (magic - 2u * Lut::kZBias)); \
        }                                                         \
    }
    EP_FIELD(1)
    EP_FIELD(2)
    EP_FIELD(3)
    EP_FIELD(4)
    EP_FIELD(5)
    EP_FIELD(6)
    EP_FIELD(7)
    EP_FIELD(8)
#undef EP_FIELD
    tl.x = x;
    if (badsym && act) corrupt = true;

    // lattice output: 2y = the bits above the magic (coordinates 1..7 of packed tables
    // carry twice their bias)
    constexpr uint32_t kLat = 0x4AC00000u + (Lut::kPacked ? 2u * Lut::kZBias : 0u);
    if (act) {
        if constexpr (RAGGED) {
            // vector g holds elements row * cols + 8q .. of a row padded to whole vectors
            const uint32_t row = (uint32_t)(g / tc.nq), q = (uint32_t)g - row * tc.nq;
            const int64_t e0 = (int64_t)row * tc.cols + 8 * (int64_t)q;
            const int n = (int)min((int64_t)8, tc.cols - 8 * (int64_t)q);
            if constexpr (DT == EP_LATTICE_I32) {
#pragma unroll
                for (int k = 0; k < 8; ++k)  // constant indices keep yb in registers
                    if (k < n) reinterpret_cast<int*>(out)[e0 + k] = (int)(yb[k] - (k < 7 ? kLat : 0x4AC00000u));
            } else {
                wf[7] = sigma * (__uint_as_float(yb[7]) - 6291456.0f);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < n) put_elem<DT>(out, e0 + k, wf[k]);
            }
        } else if constexpr (gemv_tokens<DT>() > 0) {
            // the vector's eight weights times the tokens' eight activations of its columns
            wf[7] = sigma * (__uint_as_float(yb[7]) - 6291456.0f);
            acc.madd(tc, q_now, wf);
            (void)out;
        } else if constexpr (DT == EP_LATTICE_I32) {
            int4* o = reinterpret_cast<int4*>(out) + 2 * g;
            o[0] = make_int4((int)(yb[0] - kLat), (int)(yb[1] - kLat), (int)(yb[2] - kLat), (int)(yb[3] - kLat));
            o[1] = make_int4((int)(yb[4] - kLat), (int)(yb[5] - kLat), (int)(yb[6] - kLat),
                             (int)(yb[7] - 0x4AC00000u));
        } else {
            wf[7] = sigma * (__uint_as_float(yb[7]) - 6291456.0f);
            Out<DT>::store(out, g, wf);
        }
    }
}

// Decode the tiles of this warp; the first one was begun in the prologue.

template <int DT, bool RAGGED, typename Lut>
__device__ void decode_tiles(const uint16_t* tiles, const uint32_t* tix, const float* scales, void* out,
                             const Lut& lut, const TileCtx& tc, Ring& rg, Tile& tl, uint32_t first_i) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt = lanemask_lt();
    const uint32_t G = tc.G;
    bool corrupt = false;
    bool have = tl.t != 0xFFFFFFFFu;
    GemvAcc<gemv_tokens<DT>()> acc;
    acc.init();

    for (uint32_t i = first_i; have;) {
        if (!tl.ok) {
            corrupt = true;
        } else {
            uint32_t cur = tl.off0 - tl.base;  // tile-relative word cursor
            // a3: the staging state changes only when the cursor crosses `thr`:
            // at the start of a chunk (issue the one after it) or within one round
            // of a chunk not yet waited for (wait for it)
            uint32_t thr = 0;
            // every lane's row for round 0, its row scale, and the row of round 1
            float sig_next = tl.vt > (uint32_t)lane ? __ldg(scales + tl.rowl) : 1.0f;
            acc.ahead(tc, tl.ql);
            auto round = [&](auto full, uint32_t r) {
                constexpr bool FULL = decltype(full)::value;
                if (cur >= thr) {
                    const uint32_t ci = cur >> kChunkShift;
                    if (ci + 1 < tl.nchunks && ci + 1 >= rg.seq - tl.seq0)
                        tile_issue_chunk(tiles, rg, tl, ci + 1, lane);
                    const uint32_t issued = rg.seq - tl.seq0;
                    if (issued > 0) {
                        uint32_t last = (cur + kRoundWords - 1) >> kChunkShift;
                        if (last >= issued) last = issued - 1;  // never wait on a chunk that was not issued
                        while (rg.waited - tl.seq0 <= last) ring_wait_one(rg);
                    }
                    const uint32_t nw = rg.waited - tl.seq0, ni = rg.seq - tl.seq0;
                    const uint32_t t_issue = ni < tl.nchunks ? (ni - 1) << kChunkShift : 0xFFFFFFFFu;
                    const uint32_t t_wait = nw < ni ? (nw << kChunkShift) - (kRoundWords - 1) : 0xFFFFFFFFu;
                    thr = t_issue < t_wait ? t_issue : t_wait;
                }
                uint32_t pb = rg.ring_s + 2u * ((tl.org + cur) & (kRingWords - 1));
                const uint32_t p_start = pb;
                const float sigma = sig_next;
                const uint32_t row_now = tl.rowl, q_now = tl.ql;  // this round's row and column block
                acc.enter(tc, row_now, FULL || (r << 5) + (uint32_t)lane < tl.vt);
                // advance every lane's row by 32 vectors and prefetch the next round's scale
                tl.ql += 32;
                if (tc.nq >= 32) {
                    const bool wrap = tl.ql >= tc.nq;
                    tl.ql -= wrap ? tc.nq : 0u;
                    tl.rowl += wrap ? 1u : 0u;
                } else {
                    while (tl.ql >= tc.nq) {
                        tl.ql -= tc.nq;
                        ++tl.rowl;
                    }
                }
                if (FULL) sig_next = ((r + 1) << 5) + lane < tl.vt ? __ldg(scales + tl.rowl) : 1.0f;
                decode_round<DT, RAGGED, Lut, FULL>(out, sigma, lut, tc, tl, pb, r, lt, lane, corrupt, acc, q_now);
                if (FULL) acc.ahead(tc, tl.ql);  // the next round's activations
                cur += (pb - p_start) >> 1;
            };
            for (uint32_t r = 0; r + 1 < tl.rounds; ++r) round(std::true_type{}, r);
            round(std::false_type{}, tl.rounds - 1);
            // tile end: every lane back at 2^15 and the cursor on the next offset
            if (!__all_sync(kFull, tl.x == kStateLow) || cur != tl.off1 - tl.base) corrupt = true;
            acc.warp_flush(tc, acc.pending());
            acc.init();
        }
        // drain this tile's copies before the ring is reused
        while (rg.waited < rg.seq && !rg.timed_out) ring_wait_one(rg);
        if (rg.timed_out) break;
        i += kWarps;
        const uint64_t t64 = (uint64_t)tc.cta + (uint64_t)i * G;
        have = t64 < tc.T;
        if (have) tile_begin(tc, tiles, tix, rg, tl, (uint32_t)t64, lane);
    }
    while (rg.waited < rg.seq && !rg.timed_out) ring_wait_one(rg);
    if (lane == 0) {
        unsigned bits = 0;
        if (corrupt) bits |= kStCorrupt;
        if (rg.timed_out) bits |= kStTimeout;
        if (bits) raise_status(bits);
    }
}

// ---------------------------------------------------------------- the kernel

struct Params {
    const uint16_t* tiles;
    const uint32_t* tix;
    const uint8_t* ft;
    const float* scales;
    void* out;
    uint8_t* ws;  // LUT image + grid-barrier state, or a prepared table (read only)
    int64_t rows, cols;
    uint32_t one;       // 1, set by the host (see TileCtx)
    uint32_t prepared;  // ws holds a table ep_decode_prepare wrote: no build, no grid barrier
    const uint16_t* gx;  // ep_decode_gemv: BF16 activations [tokens, cols]; the product [tokens, rows]
    float* gy;
};

// The decode loop for the stream's LUT format.  Rows padded to whole vectors (a width
// that is not a multiple of 8) run a separate kernel (RAGGED: element-wise stores), so
// the vector-store kernel is compiled without that path.
template <int DT, bool R>
__device__ __forceinline__ void run_decode(const Params& p, const Geo& g, uint32_t lut_s, const uint16_t* fq,
                                           const int* s_min, const uint32_t* s_A, const uint32_t* s_off,
                                           uint32_t desc2, const TileCtx& tc, Ring& rg, Tile& tl, uint32_t first_i) {
#define EP_PACKED(BB, FF) \
    decode_tiles<DT, R>(p.tiles, p.tix, p.scales, p.out,                                              \
                     PackedLut<BB, FF>{lut_s, tc.four, 0u - (p.one << (BB + 2))},                      \
                     tc, rg, tl, first_i)
    switch (g.mode) {
        case 9: EP_PACKED(9, false); break;
        case 10: EP_PACKED(10, false); break;
        case 11: EP_PACKED(11, false); break;
        case kModeF + 9: EP_PACKED(9, true); break;
        case kModeF + 10: EP_PACKED(10, true); break;
        case kModeF + 11: EP_PACKED(11, true); break;
        case kModeTwo:
        case kModeTwoPair: {
            const bool pair = g.mode == kModeTwoPair;
            if (pair)
                decode_tiles<DT, R>(p.tiles, p.tix, p.scales, p.out,
                                 TwoLut<true>{lut_s, g.b, g.M - 1u, g.M, desc2, s_A}, tc, rg, tl, first_i);
            else
                decode_tiles<DT, R>(p.tiles, p.tix, p.scales, p.out,
                                 TwoLut<false>{lut_s, g.b, g.M - 1u, 2u * g.M, desc2, s_A}, tc, rg, tl, first_i);
            break;
        }
        default: {
            CoarseLut cl;
            cl.lut_s = lut_s;
            cl.b = g.b;
            cl.mmask = g.M - 1;
            cl.sh = g.b - g.k;
            cl.nb_shift = g.k;
            cl.fq = fq;
            cl.s_min = s_min;
            cl.s_A = s_A;
            cl.s_off = s_off;
            decode_tiles<DT, R>(p.tiles, p.tix, p.scales, p.out, cl, tc, rg, tl, first_i);
        }
    }
#undef EP_PACKED
}

// The decode of one tensor by G CTAs, this one of rank cta (the tensor's tiles cta + i G).
// BATCH: a batch launch, always with a prepared table.
// This CTA's share of zeroing n floats (y 16-byte aligned): 16-byte stores, then the tail
__device__ __forceinline__ void zero_share(float* y, size_t n, uint32_t cta, uint32_t G) {
    const size_t n4 = n >> 2, step = (size_t)G * kThreads;
    for (size_t i = (size_t)cta * kThreads + threadIdx.x; i < n4; i += step)
        reinterpret_cast<float4*>(y)[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (cta == 0 && threadIdx.x < (n & 3u)) y[(n4 << 2) + threadIdx.x] = 0.0f;
}

template <int DT, bool RAGGED, bool BATCH>
__device__ __forceinline__ void decode_body(const Params& p, const uint32_t cta, const uint32_t G) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ int s_ok;
    int* s_min = reinterpret_cast<int*>(smem + kOffDesc);
    uint32_t* s_A = reinterpret_cast<uint32_t*>(smem + kOffDesc + 128);
    uint32_t* s_off = reinterpret_cast<uint32_t*>(smem + kOffDesc + 256);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // ep_decode_gemv with the per-call table: the product starts at zero, and the grid barrier
    // of the table build orders these stores before every CTA's first atomic add (stores issued
    // here, before the prologue's values fill the registers)
    if constexpr (gemv_tokens<DT>() > 0) {
        if (!p.prepared) zero_share(p.gy, (size_t)gemv_tokens<DT>() * (size_t)p.rows, cta, G);
    }

    // ---- prologue: header, descriptors, barriers, the first chunks of every warp's first tile
    Geo g;
    int lane_mn;
    uint32_t lane_A;
    const unsigned hs = parse_header(p.ft, p.rows, p.cols, g, lane_mn, lane_A);
    if (hs) {  // every CTA reads the same header, so every CTA leaves here
        if (threadIdx.x == 0 && cta == 0) raise_status(hs);
        return;
    }
    const bool prep = BATCH || p.prepared != 0;
    const uint16_t* fq = reinterpret_cast<const uint16_t*>(p.ft + table_header_bytes(kTables));
    // This CTA's table (one per CTA when G >= 16): its frequencies into registers now, so
    // that these loads, the coset table's, the tile records and the first payload chunks are
    // in flight together.
    uint32_t fr[kPre];
    int t_pre = 0;
    if (G >= 16 && g.mode != kModeCoarse && !prep) {
        const int t = 1 + (int)(cta * 16u / G);
        const uint32_t At = __shfl_sync(kFull, lane_A, t);
        const uint32_t offt = __reduce_add_sync(kFull, lane < t ? lane_A : 0u);
        if (At <= (uint32_t)(kPre * kThreads)) {
            t_pre = t;
#pragma unroll
            for (int k = 0; k < kPre; ++k) {
                const uint32_t q = threadIdx.x + (uint32_t)k * kThreads;
                fr[k] = q < At ? fq[offt + q] : 0u;
            }
        }
    }
    if (threadIdx.x < 32) {
        const int t = threadIdx.x;
        const uint32_t A = lane_A;
        uint32_t incl = A;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(kFull, incl, o);
            if (t >= o) incl += v;
        }
        if (t < kTables) {
            s_min[t] = lane_mn;
            s_A[t] = A;
            s_off[t] = incl - A;
        }
        // TWO: table t's records start after those of tables 1..t-1 (A + 1 each)
        const uint32_t A0 = __shfl_sync(kFull, A, 0);
        if (t >= 1 && t < kTables)
            reinterpret_cast<uint2*>(smem + kOffDesc2)[t - 1] =
                make_uint2(smem_u32(smem + kOffLut + kTwoRec) + 2u * (incl - A - A0 + (uint32_t)(t - 1)),
                           0x4AC00000u + (uint32_t)((t - 1) & 1) + (uint32_t)lane_mn * (t >= 15 ? 4u : 2u));
    }
    // a prepared table: its trailer's loads go out now, with the prologue's other loads
    uint2 fp = make_uint2(0u, 0u);
    uint4 tr4 = make_uint4(0u, 0u, 0u, 0u);
    uint32_t tr_ib = 0;
    if (prep && threadIdx.x < 32) {
        fp = table_fingerprint(g, lane_mn, lane_A);
        if (threadIdx.x == 0) {
            const uint32_t* tr = reinterpret_cast<const uint32_t*>(p.ws + kLutBytes);
            tr4 = __ldg(reinterpret_cast<const uint4*>(tr));
            tr_ib = __ldg(tr + 4);
        }
    }
    TileCtx tc;
    tc.nvec = g.nvec;
    tc.V = g.V;
    tc.T = g.T;
    tc.nq = (uint32_t)((p.cols + 7) / 8);
    tc.cols = p.cols;
    tc.gx = p.gx;
    tc.gy = p.gy;
    tc.rows = (uint32_t)p.rows;
    tc.b = g.b;
    tc.two = p.one << 1;
    tc.four = p.one << 2;
    tc.k64 = p.one << 16;
    tc.mneg = 0u - (p.one << g.b);
    tc.cta = cta;
    tc.G = G;
    // the first tile's record, in flight with the loads above and below
    Tile tl;
    tl.t = 0xFFFFFFFFu;
    const uint32_t first_i = (uint32_t)warp;
    const uint64_t t_first = (uint64_t)cta + (uint64_t)first_i * G;
    if (t_first < g.T) tile_load(tc, p.tix, tl, (uint32_t)t_first, lane);
    tc.total = p.tix[(size_t)kTileWords * g.T];
    tc.cmin = (uint32_t)__shfl_sync(kFull, lane_mn, 0);
    if (__shfl_sync(kFull, lane_A, 0) == 1u) {  // one-symbol coset table: every slot is that symbol
        tc.f0c = g.M;
        tc.f1c = 0;
    } else {
        tc.f0c = fq[0];
        tc.f1c = fq[1];
    }

    Ring rg;
    rg.ring = smem + kOffRing + warp * kRingAllocBytes;
    rg.ring_s = smem_u32(rg.ring);
    rg.bar_s = smem_u32(smem + kOffBar + warp * 16);
    rg.seq = 0;
    rg.waited = 0;
    rg.timed_out = false;
    const uint32_t lut_bar = smem_u32(smem + kOffBar + kWarps * 16);
    if (lane == 0) {
        mbar_init(rg.bar_s, 1);
        mbar_init(rg.bar_s + 8, 1);
        if (warp == 0) mbar_init(lut_bar, 1);
        fence_barrier_init();
        // a prepared image comes straight into shared memory, ahead of the payload's first chunks
        // (the copy stays inside the table buffer whatever its trailer holds; checked below)
        if (warp == 0 && prep && cta < g.T) {
            mbar_arrive_expect_tx(lut_bar, g.image_bytes);
            for (uint32_t o = 0; o < g.image_bytes; o += 16384u)
                bulk_g2s(smem_u32(smem + kOffLut) + o, p.ws + o,
                         g.image_bytes - o < 16384u ? g.image_bytes - o : 16384u, lut_bar);
        }
    }
    __syncthreads();  // barrier initialisation and descriptors visible to every warp

    if (t_first < g.T) tile_start(tc, p.tiles, rg, tl, lane);
    const bool bad_c = tc.f0c + tc.f1c != g.M;
    tc.df = tc.f1c - tc.f0c;
    tc.nf0 = 0u - tc.f0c;

    if (prep) {
        // ---- a2 from a prepared table (its copy is in flight): the trailer must carry this
        // header's layout fingerprint
        if (threadIdx.x == 0) {
            s_ok = tr4.x == kLutMagic && tr4.z == fp.x && tr4.w == fp.y && tr_ib == g.image_bytes;
            if (cta == 0 && (!s_ok || tr4.y)) raise_status(kStHeader);
        }
    } else {
        // ---- a2: this CTA's slice of the LUT image, a grid-wide arrival, the image into shared memory
        // A table that does not sum to 2^b gets zero entries (decoding with them stays in
        // bounds) and raises the status word; the decode goes on, its output unspecified.
        const bool bad = build_lut_slice(g, fq, s_min, s_A, s_off, p.ws, reinterpret_cast<uint16_t*>(smem + kOffLut),
                                         t_pre, fr);
        if (bad && threadIdx.x == 0) raise_status(kStHeader);
        fence_proxy_async_shared();  // the scratch writes before the bulk copy overwrites them
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();  // the CTA's image stores (ordered by the barrier above) before the arrival
            // the counter grows by G per launch, so the arrival that returns `old` belongs to
            // the launch that ends at the next multiple of G
            unsigned long long* arrivals = reinterpret_cast<unsigned long long*>(p.ws + kWsCountOffset);
            const unsigned long long old = atomicAdd(arrivals, 1ull);
            // old / G without a 64-bit integer division: a double quotient (old < 2^53), corrected
            const unsigned long long Gg = gridDim.x;  // the whole grid (here every CTA shares the tensor)
            unsigned long long q = (unsigned long long)((double)old / (double)Gg);
            q -= q * Gg > old ? 1ull : 0ull;
            q += (q + 1ull) * Gg <= old ? 1ull : 0ull;
            const unsigned long long target = (q + 1ull) * Gg;
            uint32_t spins = 0;
            // every CTA of the (cooperative, hence co-resident) grid arrives; bounded wait
            while (ld_acquire_gpu(arrivals) < target && spins < kGridSpins) {
                __nanosleep(32);
                ++spins;
            }
            s_ok = spins < kGridSpins;
            if (!s_ok) raise_status(kStTimeout);
            if (s_ok && cta < g.T) {
                fence_proxy_async_global();  // generic-proxy image stores before the bulk-copy reads
                mbar_arrive_expect_tx(lut_bar, g.image_bytes);
                for (uint32_t o = 0; o < g.image_bytes; o += 16384u)
                    bulk_g2s(smem_u32(smem + kOffLut) + o, p.ws + o,
                             g.image_bytes - o < 16384u ? g.image_bytes - o : 16384u, lut_bar);
            }
        }
    }
    __syncthreads();
    if (cta >= g.T) return;  // no tile for this CTA
    bool lut_ok = s_ok != 0;
    // a prepared table's copy is in flight even when its trailer did not match
    if ((lut_ok || prep) && !mbar_wait(lut_bar, 0)) {
        lut_ok = false;
        raise_status(kStTimeout);
    }
    lut_ok = __syncthreads_and(lut_ok) != 0;  // one decision for the whole CTA
    if (!lut_ok || bad_c) {
        if (bad_c && threadIdx.x == 0 && cta == 0) raise_status(kStHeader);
        while (rg.waited < rg.seq && !rg.timed_out) ring_wait_one(rg);  // drain the prologue's copies
        return;
    }

    const uint32_t lut_s = smem_u32(smem + kOffLut);
    const uint32_t desc2 = smem_u32(smem + kOffDesc2);
    run_decode<DT, RAGGED>(p, g, lut_s, fq, s_min, s_A, s_off, desc2, tc, rg, tl, first_i);
}

// With programmatic dependent launch (the prepared and batched decodes) the grid may start
// while the kernel ahead of it in the stream is ending: wait for it before any global read,
// and let the next kernel's launch go ahead (it waits the same way).  Without that launch
// attribute (the cooperative per-call decode) both are no-ops.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <int DT, bool RAGGED>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(Params p) {
    grid_dependency_wait();
    decode_body<DT, RAGGED, false>(p, blockIdx.x, gridDim.x);
}

// One CTA of a batch launch: which tensor (its arguments, a prepared table) and which share of
// its tiles.  count = 0: no work.
struct alignas(16) BatchCta {
    Params p;
    uint32_t rank, count;
};

template <int DT, bool RAGGED>
__global__ void __launch_bounds__(kThreads, 1) decode_batch_kernel(const BatchCta* plan) {
    grid_dependency_wait();
    const BatchCta c = plan[blockIdx.x];
    if (c.count == 0) return;
    decode_body<DT, RAGGED, true>(c.p, c.rank, c.count);
}

// ep_decode_prepare's kernel: a2 without the decode.  Every CTA builds its slice of the image
// into the caller's table exactly as the decode kernel builds it into the workspace; CTA 0
// writes the trailer's magic, fingerprint and image size (the host zeroed the trailer), a CTA
// that finds a table not summing to 2^b sets its bad word.
__global__ void __launch_bounds__(kThreads, 1) lut_prepare_kernel(const uint8_t* ft, int64_t rows, int64_t cols,
                                                                   uint8_t* lut) {
    extern __shared__ __align__(1024) uint8_t smem[];
    int* s_min = reinterpret_cast<int*>(smem + kPrepOffDesc);
    uint32_t* s_A = reinterpret_cast<uint32_t*>(smem + kPrepOffDesc + 128);
    uint32_t* s_off = reinterpret_cast<uint32_t*>(smem + kPrepOffDesc + 256);
    Geo g;
    int lane_mn;
    uint32_t lane_A;
    const unsigned hs = parse_header(ft, rows, cols, g, lane_mn, lane_A);
    if (hs) {
        if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(hs);
        return;
    }
    const uint16_t* fq = reinterpret_cast<const uint16_t*>(ft + table_header_bytes(kTables));
    if (threadIdx.x < 32) {
        const int t = threadIdx.x;
        uint32_t incl = lane_A;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(kFull, incl, o);
            if (t >= o) incl += v;
        }
        if (t < kTables) {
            s_min[t] = lane_mn;
            s_A[t] = lane_A;
            s_off[t] = incl - lane_A;
        }
        const uint2 fp = table_fingerprint(g, lane_mn, lane_A);
        if (t == 0 && blockIdx.x == 0) {
            uint32_t* tr = reinterpret_cast<uint32_t*>(lut + kLutBytes);
            tr[0] = kLutMagic;
            tr[2] = fp.x;
            tr[3] = fp.y;
            tr[4] = g.image_bytes;
        }
    }
    __syncthreads();
    uint32_t fr[kPre] = {};
    const bool bad = build_lut_slice(g, fq, s_min, s_A, s_off, lut, reinterpret_cast<uint16_t*>(smem), 0, fr);
    if (bad && threadIdx.x == 0) {
        raise_status(kStHeader);
        atomicOr(reinterpret_cast<unsigned*>(lut + kLutBytes) + 1, 1u);
    }
}

// ------------------------------------------------------------- host side

struct DevState {
    int num_sms = 0;
    bool attr_done[8] = {};
    bool prep_attr_done = false;
    bool gemv_attr_done = false;
    uint8_t* ws = nullptr;         // the LUT workspace of this device
    cudaEvent_t ws_free = nullptr;  // recorded after every decode that used it
};
DevState g_dev[64];
std::mutex g_mu;

template <int DT>
cudaError_t set_decode_attr() {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<DT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(decode_kernel<DT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(decode_batch_kernel<DT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(decode_batch_kernel<DT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
    return e;
}

cudaError_t dev_setup(int dev, int dt, DevState*& ds, bool need_ws = true) {
    std::lock_guard<std::mutex> lk(g_mu);
    ds = &g_dev[dev];
    cudaError_t e;
    if (!ds->num_sms) {
        e = cudaDeviceGetAttribute(&ds->num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    if (need_ws && !ds->ws) {
        // one workspace per device, zeroed once; the grid barrier in it resets itself
        void* w = nullptr;
        e = cudaMalloc(&w, kWsBytes);
        if (e != cudaSuccess) return e;
        e = cudaMemset(w, 0, kWsBytes);
        if (e != cudaSuccess) return e;
        e = cudaEventCreateWithFlags(&ds->ws_free, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        ds->ws = static_cast<uint8_t*>(w);
    }
    if (!ds->attr_done[dt]) {
        switch (dt) {
            case EP_BF16: e = set_decode_attr<EP_BF16>(); break;
            case EP_FP16: e = set_decode_attr<EP_FP16>(); break;
            case EP_FP8_E4M3: e = set_decode_attr<EP_FP8_E4M3>(); break;
            case EP_INT8: e = set_decode_attr<EP_INT8>(); break;
            case EP_UINT8: e = set_decode_attr<EP_UINT8>(); break;
            case EP_FP32: e = set_decode_attr<EP_FP32>(); break;
            default: e = set_decode_attr<EP_LATTICE_I32>(); break;
        }
        if (e != cudaSuccess) return e;
        ds->attr_done[dt] = true;
    }
    return cudaSuccess;
}

// ep_decode_gemv's kernels (widths that are a multiple of 8 only)
template <int NT>
cudaError_t set_gemv_attr() {
    return cudaFuncSetAttribute(decode_kernel<kGemv + NT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemBytes);
}

template <int DT>
cudaError_t launch_decode(const Params& prm, cudaStream_t st, int num_sms) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_sms);  // one CTA per SM
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (prm.prepared) {
        // a prepared table needs no grid barrier: an ordinary launch that may be scheduled
        // while the kernel ahead of it in the stream ends (programmatic dependent launch)
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    } else {
        // the grid barrier needs every CTA co-resident (a cooperative launch)
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return (prm.cols & 7) ? cudaLaunchKernelEx(&cfg, decode_kernel<DT, true>, prm)
                          : cudaLaunchKernelEx(&cfg, decode_kernel<DT, false>, prm);
}

// ep_decode_gemv: NT tokens; cooperative with the grid-built table, or an ordinary launch with
// programmatic dependent launch when a prepared table is given (as launch_decode)
template <int NT>
cudaError_t launch_gemv_nt(const Params& prm, cudaStream_t st, int num_sms) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)num_sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (prm.prepared) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    } else {
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<kGemv + NT, false>, prm);
}

cudaError_t launch_gemv(int ntok, const Params& prm, cudaStream_t st, int num_sms) {
    switch (ntok) {
        case 1: return launch_gemv_nt<1>(prm, st, num_sms);
        case 2: return launch_gemv_nt<2>(prm, st, num_sms);
        case 4: return launch_gemv_nt<4>(prm, st, num_sms);
        default: return launch_gemv_nt<8>(prm, st, num_sms);
    }
}

cudaError_t launch_any(ep_dtype dt, const Params& prm, cudaStream_t st, int num_sms) {
    switch (dt) {
        case EP_BF16: return launch_decode<EP_BF16>(prm, st, num_sms);
        case EP_FP16: return launch_decode<EP_FP16>(prm, st, num_sms);
        case EP_FP8_E4M3: return launch_decode<EP_FP8_E4M3>(prm, st, num_sms);
        case EP_INT8: return launch_decode<EP_INT8>(prm, st, num_sms);
        case EP_UINT8: return launch_decode<EP_UINT8>(prm, st, num_sms);
        case EP_FP32: return launch_decode<EP_FP32>(prm, st, num_sms);
        default: return launch_decode<EP_LATTICE_I32>(prm, st, num_sms);
    }
}

template <int DT>
cudaError_t launch_batch(const BatchCta* plan, int ctas, bool ragged, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);  // one CTA per SM; an ordinary launch (no grid barrier)
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // as a prepared decode
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return ragged ? cudaLaunchKernelEx(&cfg, decode_batch_kernel<DT, true>, plan)
                  : cudaLaunchKernelEx(&cfg, decode_batch_kernel<DT, false>, plan);
}

cudaError_t launch_batch_any(ep_dtype dt, const BatchCta* plan, int ctas, bool ragged, cudaStream_t st) {
    switch (dt) {
        case EP_BF16: return launch_batch<EP_BF16>(plan, ctas, ragged, st);
        case EP_FP16: return launch_batch<EP_FP16>(plan, ctas, ragged, st);
        case EP_FP8_E4M3: return launch_batch<EP_FP8_E4M3>(plan, ctas, ragged, st);
        case EP_INT8: return launch_batch<EP_INT8>(plan, ctas, ragged, st);
        case EP_UINT8: return launch_batch<EP_UINT8>(plan, ctas, ragged, st);
        case EP_FP32: return launch_batch<EP_FP32>(plan, ctas, ragged, st);
        default: return launch_batch<EP_LATTICE_I32>(plan, ctas, ragged, st);
    }
}

// A model of one tensor's decode time on c CTAs (arbitrary units), for sharing out the SMs:
// a sub-partition either issues its share of the steps (about 31 instructions a step with a
// packed table, more with the two-level or bucketed ones at b >= 12) or, with few tiles a warp,
// waits on their chains (about 158 cycles a step, at least one tile a warp).  Continuous in c,
// so that every further CTA lowers it.
double batch_time(int64_t T, int64_t V, int b, int64_t c) {
    const double steps = (double)((V + 31) / 32) * 9.0;
    const double per_cta = (double)T / (double)c;
    const double per_warp = per_cta / kWarps > 1.0 ? per_cta / kWarps : 1.0;
    const double issue = per_cta / 4.0 * steps * (b >= 12 ? 48.0 : 31.4);
    const double chain = per_warp * steps * 158.0;
    return issue > chain ? issue : chain;
}

bool misaligned(const void* q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) != 0; }

// A launch that builds the table in the device's workspace: it waits (on the GPU) for the
// previous such launch, whatever stream that ran on (not applied while the stream is being
// captured), and marks the workspace busy until it ends.
template <typename Launch>
ep_status workspace_launch(DevState* ds, cudaStream_t st, Launch launch) {
    std::lock_guard<std::mutex> lk(g_mu);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cap);
    const bool capturing = e == cudaSuccess && cap != cudaStreamCaptureStatusNone;
    if (e == cudaSuccess && !capturing) e = cudaStreamWaitEvent(st, ds->ws_free, 0);
    if (e == cudaSuccess) e = launch(st);
    if (e == cudaSuccess && !capturing) e = cudaEventRecord(ds->ws_free, st);
    return e == cudaSuccess ? EP_OK : EP_ECUDA;
}

// the host checks every decode entry point shares
ep_status check_decode_args(const uint16_t* tiles, const uint32_t* tile_index, const uint8_t* freq_tables,
                            const float* row_scales, int64_t rows, int64_t cols, ep_dtype out_dtype, void* out) {
    if (!tiles || !tile_index || !freq_tables || !row_scales || !out) return EP_EINVAL;
    if (rows <= 0 || cols <= 0) return EP_EINVAL;
    if ((int)out_dtype < EP_BF16 || (int)out_dtype > EP_UINT8) return EP_EUNSUPPORTED;
    // the largest tensor: fewer than 2^31 vectors of eight (each factor bounded first, so that
    // the product cannot overflow)
    if (rows >= (1ll << 31) || cols >= (1ll << 34)) return EP_EINVAL;
    const int64_t nvec = rows * ((cols + 7) / 8);
    if (nvec >= (1ll << 31)) return EP_EINVAL;
    if (misaligned(tiles, 16) || misaligned(freq_tables, 16) || misaligned(tile_index, 4) ||
        misaligned(row_scales, 4) || misaligned(out, 16))
        return EP_EINVAL;
    return EP_OK;
}

}  // namespace
}  // namespace ep

extern "C" {

ep_status ep_decode_tensor(void* stream, const uint16_t* tiles, const uint32_t* tile_index,
                           const uint8_t* freq_tables, const float* row_scales, int64_t rows, int64_t cols,
                           ep_dtype out_dtype, void* out) {
    using namespace ep;
    const ep_status as = check_decode_args(tiles, tile_index, freq_tables, row_scales, rows, cols, out_dtype, out);
    if (as != EP_OK) return as;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EP_ECUDA;
    DevState* ds = nullptr;
    if (dev_setup(dev, (int)out_dtype, ds) != cudaSuccess) return EP_ECUDA;
    const Params prm{tiles, tile_index, freq_tables, row_scales, out, ds->ws, rows, cols, 1u, 0u};
    return workspace_launch(ds, static_cast<cudaStream_t>(stream),
                            [&](cudaStream_t st) { return launch_any(out_dtype, prm, st, ds->num_sms); });
}

ep_status ep_decode_prepare(void* stream, const uint8_t* freq_tables, int64_t rows, int64_t cols, void* lut,
                            size_t lut_bytes) {
    using namespace ep;
    if (!freq_tables || !lut || lut_bytes < (size_t)EP_LUT_BYTES || rows <= 0 || cols <= 0) return EP_EINVAL;
    if (misaligned(freq_tables, 16) || misaligned(lut, 16)) return EP_EINVAL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EP_ECUDA;
    DevState* ds = nullptr;
    if (dev_setup(dev, EP_BF16, ds, false) != cudaSuccess) return EP_ECUDA;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!ds->prep_attr_done) {
            if (cudaFuncSetAttribute(lut_prepare_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kPrepSmemBytes) != cudaSuccess)
                return EP_ECUDA;
            ds->prep_attr_done = true;
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* l = static_cast<uint8_t*>(lut);
    cudaError_t e = cudaMemsetAsync(l + kLutBytes, 0, EP_LUT_BYTES - kLutBytes, st);
    if (e == cudaSuccess) {
        lut_prepare_kernel<<<ds->num_sms, kThreads, kPrepSmemBytes, st>>>(freq_tables, rows, cols, l);
        e = cudaGetLastError();
    }
    return e == cudaSuccess ? EP_OK : EP_ECUDA;
}

ep_status ep_decode_tensor_prepared(void* stream, const uint16_t* tiles, const uint32_t* tile_index,
                                    const uint8_t* freq_tables, const float* row_scales, const void* lut,
                                    size_t lut_bytes, int64_t rows, int64_t cols, ep_dtype out_dtype,
                                    void* out) {
    using namespace ep;
    const ep_status as = check_decode_args(tiles, tile_index, freq_tables, row_scales, rows, cols, out_dtype, out);
    if (as != EP_OK) return as;
    if (!lut || lut_bytes < (size_t)EP_LUT_BYTES || misaligned(lut, 16)) return EP_EINVAL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EP_ECUDA;
    DevState* ds = nullptr;
    if (dev_setup(dev, (int)out_dtype, ds, false) != cudaSuccess) return EP_ECUDA;
    // the table is only read: no workspace, nothing to order against other decodes
    const Params prm{tiles, tile_index, freq_tables, row_scales, out,
                     const_cast<uint8_t*>(static_cast<const uint8_t*>(lut)), rows, cols, 1u, 1u};
    return launch_any(out_dtype, prm, static_cast<cudaStream_t>(stream), ds->num_sms) == cudaSuccess ? EP_OK
                                                                                                     : EP_ECUDA;
}

ep_status ep_decode_gemv(void* stream, const uint16_t* tiles, const uint32_t* tile_index, const uint8_t* freq_tables,
                         const float* row_scales, const void* lut, size_t lut_bytes, int64_t rows, int64_t cols,
                         const void* x, int ntok, float* y) {
    using namespace ep;
    const ep_status as = check_decode_args(tiles, tile_index, freq_tables, row_scales, rows, cols, EP_FP32, y);
    if (as != EP_OK) return as;
    if (!x || misaligned(x, 16)) return EP_EINVAL;
    if (ntok != 1 && ntok != 2 && ntok != 4 && ntok != 8) return EP_EUNSUPPORTED;
    if (cols & 7) return EP_EUNSUPPORTED;
    if (lut && (lut_bytes < (size_t)EP_LUT_BYTES || misaligned(lut, 16))) return EP_EINVAL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EP_ECUDA;
    DevState* ds = nullptr;
    if (dev_setup(dev, EP_FP32, ds) != cudaSuccess) return EP_ECUDA;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!ds->gemv_attr_done) {
            if (set_gemv_attr<1>() != cudaSuccess || set_gemv_attr<2>() != cudaSuccess ||
                set_gemv_attr<4>() != cudaSuccess || set_gemv_attr<8>() != cudaSuccess)
                return EP_ECUDA;
            ds->gemv_attr_done = true;
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (lut) {
        // the product accumulates by atomic adds: it starts at zero (with the per-call table the
        // kernel zeroes it before its grid barrier)
        if (cudaMemsetAsync(y, 0, (size_t)ntok * (size_t)rows * sizeof(float), st) != cudaSuccess) return EP_ECUDA;
        const Params prm{tiles, tile_index, freq_tables, row_scales, y,
                         const_cast<uint8_t*>(static_cast<const uint8_t*>(lut)), rows, cols, 1u, 1u,
                         static_cast<const uint16_t*>(x), y};
        return launch_gemv(ntok, prm, st, ds->num_sms) == cudaSuccess ? EP_OK : EP_ECUDA;
    }
    const Params prm{tiles, tile_index, freq_tables, row_scales, y, ds->ws, rows, cols, 1u, 0u,
                     static_cast<const uint16_t*>(x), y};
    return workspace_launch(ds, st, [&](cudaStream_t s2) { return launch_gemv(ntok, prm, s2, ds->num_sms); });
}

ep_status ep_batch_apportion(int n, const int64_t* ntiles, const int64_t* tile_vectors, const int* prob_bits,
                             int num_ctas, int* counts) {
    using namespace ep;
    if (n <= 0 || !ntiles || !tile_vectors || !prob_bits || !counts || num_ctas < n) return EP_EINVAL;
    for (int k = 0; k < n; ++k) {
        if (ntiles[k] < 1 || tile_vectors[k] < 1) return EP_EINVAL;
        counts[k] = 1;
    }
    // each further CTA goes to the tensor that would finish last, while it has a tile for it
    for (int c = n; c < num_ctas; ++c) {
        int best = -1;
        double bt = -1.0;
        for (int k = 0; k < n; ++k) {
            if (counts[k] >= ntiles[k]) continue;
            const double t = batch_time(ntiles[k], tile_vectors[k], prob_bits[k], counts[k]);
            if (t > bt) {
                bt = t;
                best = k;
            }
        }
        if (best < 0) break;
        ++counts[best];
    }
    return EP_OK;
}

}  // extern "C"

struct ep_batch {
    int dev;
    int ctas;
    ep_dtype dt;
    bool ragged;
    ep::BatchCta* plan;  // device, one entry per CTA
};

extern "C" {

ep_status ep_batch_create(const ep_batch_item* items, int n_items, ep_dtype out_dtype, ep_batch** out) {
    return ep_batch_create_on(items, n_items, out_dtype, 0, out);
}

ep_status ep_batch_create_on(const ep_batch_item* items, int n_items, ep_dtype out_dtype, int num_ctas,
                             ep_batch** out) {
    using namespace ep;
    if (!items || !out || n_items <= 0 || num_ctas < 0) return EP_EINVAL;
    *out = nullptr;
    if ((int)out_dtype < EP_BF16 || (int)out_dtype > EP_UINT8) return EP_EUNSUPPORTED;
    bool ragged = false;
    for (int k = 0; k < n_items; ++k) {
        const ep_batch_item& it = items[k];
        const ep_status as = check_decode_args(it.tiles, it.tile_index, it.freq_tables, it.row_scales, it.rows,
                                               it.cols, out_dtype, it.out);
        if (as != EP_OK) return as;
        if (!it.lut || misaligned(it.lut, 16) || it.ntiles < 1 || it.tile_vectors < 1) return EP_EINVAL;
        ragged |= (it.cols & 7) != 0;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EP_ECUDA;
    DevState* ds = nullptr;
    if (dev_setup(dev, (int)out_dtype, ds, false) != cudaSuccess) return EP_ECUDA;
    const int nctas = num_ctas == 0 ? ds->num_sms : num_ctas;
    if (nctas > ds->num_sms) return EP_EINVAL;  // at most one CTA per SM
    if (n_items > nctas) return EP_EINVAL;      // at most one tensor per SM
    std::vector<int64_t> T(n_items), V(n_items);
    std::vector<int> b(n_items), counts(n_items);
    for (int k = 0; k < n_items; ++k) {
        T[k] = items[k].ntiles;
        V[k] = items[k].tile_vectors;
        b[k] = items[k].prob_bits;
    }
    if (ep_batch_apportion(n_items, T.data(), V.data(), b.data(), nctas, counts.data()) != EP_OK)
        return EP_EINVAL;
    std::vector<BatchCta> plan((size_t)nctas);
    size_t c = 0;
    for (int k = 0; k < n_items; ++k) {
        const ep_batch_item& it = items[k];
        const Params prm{it.tiles, it.tile_index, it.freq_tables, it.row_scales, it.out,
                         const_cast<uint8_t*>(static_cast<const uint8_t*>(it.lut)), it.rows, it.cols, 1u, 1u};
        for (int r = 0; r < counts[k]; ++r, ++c) plan[c] = BatchCta{prm, (uint32_t)r, (uint32_t)counts[k]};
    }
    for (; c < plan.size(); ++c) plan[c] = BatchCta{};  // count 0: no work
    ep_batch* h = new (std::nothrow) ep_batch{dev, nctas, out_dtype, ragged, nullptr};
    if (!h) return EP_ENOMEM;
    void* d = nullptr;
    if (cudaMalloc(&d, plan.size() * sizeof(BatchCta)) != cudaSuccess) {
        delete h;
        return EP_ECUDA;
    }
    if (cudaMemcpy(d, plan.data(), plan.size() * sizeof(BatchCta), cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(d);
        delete h;
        return EP_ECUDA;
    }
    h->plan = static_cast<BatchCta*>(d);
    *out = h;
    return EP_OK;
}

ep_status ep_decode_batch(void* stream, const ep_batch* batch) {
    using namespace ep;
    if (!batch || !batch->plan) return EP_EINVAL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return EP_ECUDA;
    if (dev != batch->dev) return EP_EINVAL;
    return launch_batch_any(batch->dt, batch->plan, batch->ctas, batch->ragged, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? EP_OK
               : EP_ECUDA;
}

void ep_batch_free(ep_batch* batch) {
    if (!batch) return;
    if (batch->plan) cudaFree(batch->plan);
    delete batch;
}

ep_status ep_decode_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned int v = 0;
    const unsigned int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&v, ep::g_decode_status, sizeof(v), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return EP_ECUDA;
    if (cudaMemcpyToSymbolAsync(ep::g_decode_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) !=
        cudaSuccess)
        return EP_ECUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return EP_ECUDA;
    if (v & ep::kStTimeout) {
        // a wait that ran out may leave the grid barrier half-counted: start it afresh
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
            std::lock_guard<std::mutex> lk(ep::g_mu);
            if (ep::g_dev[dev].ws &&
                cudaMemset(ep::g_dev[dev].ws + ep::kWsCountOffset, 0, ep::kWsBytes - ep::kWsCountOffset) !=
                    cudaSuccess)
                return EP_ECUDA;
        }
    }
    if (v & (ep::kStHeader | ep::kStCorrupt | ep::kStTimeout)) return EP_ECORRUPT;
    if (v & ep::kStUnsupported) return EP_EUNSUPPORTED;
    return EP_OK;
}

const char* ep_status_string(ep_status s) {
    switch (s) {
        case EP_OK: return "ok";
        case EP_EINVAL: return "invalid argument";
        case EP_EUNSUPPORTED: return "unsupported";
        case EP_EALPHABET: return "alphabet does not fit the precision";
        case EP_ECUDA: return "CUDA error";
        case EP_ECORRUPT: return "corrupt stream or table header";
        case EP_ENOMEM: return "out of host memory";
    }
    return "unknown status";
}

}  // extern "C"

// ----------------------------------------------- decode without allocation
//
// ep_decode_tensor_noalloc: the same decode, with its scratch (the decode
// lookup-table image and the grid-barrier words) in a file-scope device array
// instead of the workspace ep_decode_tensor allocates.  The array is a
// host-side stand-in in host code: its device address is taken with
// cudaGetSymbolAddress once per device, with that device current, on the
// first call there.

namespace ep {
namespace {

// 128 KiB of lookup-table image (the largest any stream needs, b <= 15) plus
// the 32 bytes of barrier state; every GPU that loads the library keeps it.
constexpr size_t kNoAllocScratchBytes = (size_t)kWsBytes;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
static_assert(kLutBytes + 32 <= (int)kNoAllocScratchBytes, "scratch array too small for the table image");

struct NoAllocState {
    int num_sms = 0;
    bool attr_done[8] = {};
    uint8_t* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};
NoAllocState g_noalloc[64];
std::mutex g_noalloc_mu;

cudaError_t noalloc_setup(int dev, int dt, NoAllocState*& ns) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    ns = &g_noalloc[dev];
    cudaError_t e;
    if (!ns->num_sms) {
        e = cudaDeviceGetAttribute(&ns->num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    if (!ns->scratch) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        ns->scratch = static_cast<uint8_t*>(ptr);
    }
    if (!ns->attr_done[dt]) {
        switch (dt) {
            case EP_BF16: e = set_decode_attr<EP_BF16>(); break;
            case EP_FP16: e = set_decode_attr<EP_FP16>(); break;
            case EP_FP8_E4M3: e = set_decode_attr<EP_FP8_E4M3>(); break;
            case EP_INT8: e = set_decode_attr<EP_INT8>(); break;
            case EP_UINT8: e = set_decode_attr<EP_UINT8>(); break;
            case EP_FP32: e = set_decode_attr<EP_FP32>(); break;
            default: e = set_decode_attr<EP_LATTICE_I32>(); break;
        }
        if (e != cudaSuccess) return e;
        ns->attr_done[dt] = true;
    }
    return cudaSuccess;
}

}  // namespace
}  // namespace ep

extern "C" ep_status ep_decode_tensor_noalloc(void* stream, const uint16_t* tiles, const uint32_t* tile_index,
                                              const uint8_t* freq_tables, const float* row_scales, int64_t rows,
                                              int64_t cols, ep_dtype out_dtype, void* out) {
    using namespace ep;
    // the largest tensor this entry point takes: fewer than 2^31 vectors of eight
    const ep_status as = check_decode_args(tiles, tile_index, freq_tables, row_scales, rows, cols, out_dtype, out);
    if (as != EP_OK) return as;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EP_ECUDA;
    NoAllocState* ns = nullptr;
    if (noalloc_setup(dev, (int)out_dtype, ns) != cudaSuccess) return EP_ECUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the barrier words must start at zero; the array keeps whatever the last call left
    cudaError_t e = cudaMemsetAsync(ns->scratch + kWsCountOffset, 0, kNoAllocScratchBytes - kWsCountOffset, st);
    if (e == cudaSuccess) {
        const Params prm{tiles, tile_index, freq_tables, row_scales, out, ns->scratch, rows, cols, 1u, 0u};
        e = launch_any(out_dtype, prm, st, ns->num_sms);
    }
    return e == cudaSuccess ? EP_OK : EP_ECUDA;
}
