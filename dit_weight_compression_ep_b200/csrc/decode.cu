// decode.cu -- fused EntroPack weight reconstruction for B200 (sm_100a).
//
// One launch decodes a whole tensor (EntroPack paper, Fig. 2b: symbol decode,
// lattice reconstruction, row rescaling and dtype conversion fused on the GPU;
// §3.6 "one tile to a GPU warp and one state to each lane"; App. C.3).
//
// Grid: one persistent CTA of 32 warps per SM.  Tile t goes to CTA t mod G; the
// CTA's i-th tile goes to warp i mod 32, so every SM gets within one tile of the
// same work.  Per CTA:
//   a2  the 16 coordinate tables become decode LUTs in shared memory:
//       PACKED (b <= 11, |z| small): one 32-bit entry per slot,
//         [bias = slot - cum : b][f - 1 : b][z : 32 - 2b, signed], one LDS per symbol;
//       COARSE (any b): one 64-bit entry per bucket of 2^(b-k) slots,
//         {cum | f << 16, z}, plus a short forward walk over global frequencies.
//       The coset table (2 symbols) needs no LUT: a compare picks c.
// Per warp and tile:
//   a1  32 terminal states (one per lane) and the payload offsets;
//   a3  payload words staged by cp.async.bulk (TMA 1-D) into a double-buffered
//       ring of 2 x 512 words; each chunk landing in the first half is also
//       copied to a 288-word mirror after the ring, so one round (at most 288
//       words) never needs to wrap an index;
//   a4  per round r: every lane decodes the 9 fields of vector 32r + lane
//       (c, z1..z7, m); the lanes that renormalise read consecutive words in
//       ascending lane order (ballot + popc);
//   a5  z8 = 2m + parity(z1..z7); y = z + c/2;
//   a6  w = fl32(sigma_row * y) as one FFMA: fma(sigma, z, c ? sigma/2 : -0),
//       exact to a single rounding because sigma/2 is exact;
//   a7  conversion (cvt.rn bf16x2 / f16x2, satfinite e4m3x2, rni + clamp for
//       int8) and one 16-byte (8-byte for 8-bit outputs) store per lane, so a
//       warp writes 512 (256) contiguous bytes per round.
// Stream errors never fault or trap: every shared-memory index is masked or
// bounded, every global read stays inside the buffers the header describes, and
// inconsistencies raise bits in a device status word read by ep_decode_status.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "entropack.h"
#include "ep_format.h"

namespace ep {
namespace {

constexpr int kWarps = 32;
constexpr int kThreads = 32 * kWarps;
constexpr int kChunkWords = 512;                 // words per staged chunk
constexpr int kChunkShift = 9;
constexpr int kRingWords = 2 * kChunkWords;      // double buffer
constexpr int kRoundWords = kFields * kLanes;    // 288: most words one round can consume
constexpr int kRingAllocBytes = 2688;            // (1024 + 288) words, rounded up to 128 bytes
constexpr int kCoarseBits = 10;                  // COARSE: 2^10 buckets per table

// shared-memory layout (bytes)
constexpr int kLutBytes = 128 * 1024;
constexpr int kOffLut = 0;
constexpr int kOffRing = kOffLut + kLutBytes;
constexpr int kOffBar = kOffRing + kWarps * kRingAllocBytes;
constexpr int kOffDesc = kOffBar + kWarps * 16;
constexpr int kOffFlag = kOffDesc + 3 * 32 * 4;
constexpr int kSmemBytes = kOffFlag + 16;

// status bits
constexpr unsigned kStCorrupt = 1u;      // payload / state / offset inconsistent
constexpr unsigned kStHeader = 2u;       // table header or tables invalid
constexpr unsigned kStUnsupported = 4u;  // a format variant this decoder does not handle
constexpr unsigned kStTimeout = 8u;      // a bulk copy did not complete in time

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr uint32_t kWaitSpins = 1u << 20;  // bound on mbarrier polls (each poll may suspend)

}  // namespace

__device__ unsigned int g_decode_status;

namespace {

enum : int { kModePacked9 = 9, kModePacked10 = 10, kModePacked11 = 11, kModeCoarse = 1 };

struct Params {
    const uint16_t* tiles;
    const uint32_t* tix;
    const uint8_t* ft;
    const float* scales;
    void* out;
    int64_t rows, cols;
};

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
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds_u64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ void raise_status(unsigned bits) { atomicOr(&g_decode_status, bits); }

// ------------------------------------------------------ per-warp payload ring

struct Ring {
    uint32_t ring_s;  // shared address of this warp's ring
    uint32_t bar_s;   // shared address of its two mbarriers
    uint32_t seq;     // chunks issued by this warp so far (all tiles)
    uint32_t waited;  // chunks waited for so far
    bool timed_out;
};

// Issue chunk `seq_no` of the current tile: words [src, src + n) into ring half
// seq_no & 1 (and its first 288 words to the mirror when it is the first half).
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
    const uint32_t bar = rg.bar_s + 8u * (s & 1u);
    const uint32_t parity = (s >> 1) & 1u;
    uint32_t spins = 0;
    while (!mbar_try_wait(bar, parity)) {
        if (++spins > kWaitSpins) {
            rg.timed_out = true;
            break;
        }
    }
    rg.waited = s + 1;
}

// ------------------------------------------------------------ output writers

template <int DT>
struct Out;

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
template <>
struct Out<EP_INT8> {
    __device__ static void store(void* out, int64_t g, const float w[8]) {
        int q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = __float2int_rn(fminf(fmaxf(w[i], -127.0f), 127.0f));
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

// PACKED: 16 tables x 2^B slots x 32-bit entries at lut_s; table (2(k-1) + c).
template <int B>
struct PackedLut {
    static constexpr uint32_t kM = 1u << B;
    uint32_t lut_s;
    __device__ __forceinline__ uint32_t coset_base(int c) const { return lut_s + ((uint32_t)c << (B + 2)); }
    // Decode one coordinate symbol of field k (1..8) for the coset base cb.
    template <int K>
    __device__ __forceinline__ int decode(uint32_t& x, uint32_t cb, bool& bad) const {
        const uint32_t slot = x & (kM - 1);
        const uint32_t e = lds_u32(cb + (uint32_t)(2 * (K - 1)) * (kM * 4u) + slot * 4u);
        const uint32_t bias = e & (kM - 1);
        const uint32_t fm1 = (e >> B) & (kM - 1);
        const uint32_t xs = x >> B;
        x = fm1 * xs + (xs + bias);
        (void)bad;
        return static_cast<int>(e) >> (2 * B);
    }
};

// COARSE: 16 tables x 2^k buckets x 64-bit {cum | f << 16, z}; runtime b.
struct CoarseLut {
    uint32_t lut_s;
    uint32_t b, mmask, sh, nb_shift;  // bucket = slot >> sh; table stride = 8 << nb_shift
    const uint16_t* fq;               // global frequencies
    const int* s_min;
    const uint32_t* s_A;
    const uint32_t* s_off;
    __device__ __forceinline__ uint32_t coset_base(int c) const { return lut_s + ((uint32_t)c << (nb_shift + 3)); }
    template <int K>
    __device__ __forceinline__ int decode(uint32_t& x, uint32_t cb, bool& bad) const {
        const uint32_t slot = x & mmask;
        const uint2 e = lds_u64(cb + (uint32_t)(2 * (K - 1)) * (8u << nb_shift) + (slot >> sh) * 8u);
        uint32_t c0 = e.x & 0xFFFFu, f = e.x >> 16;
        int z = static_cast<int>(e.y);
        if (slot >= c0 + f) {
            // table index of this lane: from the coset base
            const int t = 1 + 2 * (K - 1) + (int)((cb - lut_s) >> (nb_shift + 3));
            const int mn = s_min[t];
            const uint32_t A = s_A[t], off = s_off[t];
            // the walk may cross zero-frequency symbols (unobserved values inside
            // the alphabet), so it is bounded by the alphabet, not by the bucket width
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
        return z;
    }
};

// ------------------------------------------------------------- LUT builders

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// PACKED build.  Phase 1 (warps 0..15, table w+1): cumulative frequencies into a
// u16 scratch area of shared memory and, per 32-slot block, the symbol holding
// the block's first slot.  Phase 2 (all threads): entries of 4 consecutive slots
// per thread, written as one 16-byte store (a warp writes 512 contiguous bytes).
template <int B>
__device__ void build_packed(uint8_t* smem, const uint16_t* fq, const int* s_min, const uint32_t* s_A,
                             const uint32_t* s_off, volatile int* s_bad) {
    constexpr uint32_t M = 1u << B;
    constexpr uint32_t kBlocks = M / 32;
    uint16_t* cum_all = reinterpret_cast<uint16_t*>(smem + kOffRing);
    uint16_t* blk_all = cum_all + 16 * (M + 1);  // cum area sized for A <= M per table
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < 16) {
        const int t = warp + 1;
        const uint32_t A = s_A[t], off = s_off[t];
        uint16_t* cum = cum_all + (t - 1) * (M + 1);
        uint16_t* blk = blk_all + (t - 1) * kBlocks;
        uint32_t carry = 0;
        for (uint32_t base = 0; base < A; base += 32) {
            const uint32_t s = base + lane;
            const uint32_t f = s < A ? fq[off + s] : 0u;
            const uint32_t incl = warp_incl_scan(f, lane);
            const uint32_t c0 = carry + incl - f;
            if (s < A) cum[s] = (uint16_t)(c0 < M ? c0 : M);
            if (f > 0 && c0 < M) {
                uint32_t end = c0 + f < M ? c0 + f : M;
                for (uint32_t j = (c0 + 31) >> 5; (j << 5) < end; ++j) blk[j] = (uint16_t)s;
            }
            carry += __shfl_sync(kFull, incl, 31);
        }
        if (lane == 0) {
            cum[A] = (uint16_t)(carry <= M ? carry : M);
            if (A > 0 && carry != M) *s_bad = 1;
        }
    }
    __syncthreads();
    if (*s_bad) return;
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + kOffLut);
    for (uint32_t q = threadIdx.x; q < 16u * (M / 4); q += kThreads) {
        const int t = (int)(q / (M / 4)) + 1;
        const uint32_t slot0 = (q % (M / 4)) * 4;
        const uint32_t A = s_A[t];
        uint4 v = make_uint4(0, 0, 0, 0);
        if (A > 0) {
            const uint16_t* cum = cum_all + (t - 1) * (M + 1);
            const uint16_t* blk = blk_all + (t - 1) * kBlocks;
            const int mn = s_min[t];
            uint32_t s = blk[slot0 >> 5];
            uint32_t e[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t slot = slot0 + k;
                while (s + 1 < A && cum[s + 1] <= slot) ++s;
                const uint32_t c0 = cum[s], f = cum[s + 1] - c0;
                e[k] = (slot - c0) | ((f - 1) << B) | ((uint32_t)((int)s + mn) << (2 * B));
            }
            v = make_uint4(e[0], e[1], e[2], e[3]);
        }
        reinterpret_cast<uint4*>(lut)[q] = v;
    }
}

// COARSE build (warps 0..15, table w+1): bucket j of 2^sh slots holds the symbol
// that owns slot j << sh, with its cum, f and value.
__device__ void build_coarse(uint8_t* smem, const uint16_t* fq, uint32_t b, uint32_t sh, uint32_t nb_shift,
                             const int* s_min, const uint32_t* s_A, const uint32_t* s_off, volatile int* s_bad) {
    const uint32_t M = 1u << b;
    const uint32_t NB = 1u << nb_shift;
    uint2* lut = reinterpret_cast<uint2*>(smem + kOffLut);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp >= 16) return;
    const int t = warp + 1;
    const uint32_t A = s_A[t], off = s_off[t];
    const int mn = s_min[t];
    uint2* tl = lut + (size_t)(t - 1) * NB;
    if (A == 0) {
        for (uint32_t j = lane; j < NB; j += 32) tl[j] = make_uint2(0u, 0u);
        return;
    }
    uint32_t carry = 0;
    for (uint32_t base = 0; base < A; base += 32) {
        const uint32_t s = base + lane;
        const uint32_t f = s < A ? fq[off + s] : 0u;
        const uint32_t incl = warp_incl_scan(f, lane);
        const uint32_t c0 = carry + incl - f;
        if (f > 0 && c0 < M) {
            const uint32_t end = c0 + f < M ? c0 + f : M;
            const uint32_t w = 1u << sh;
            for (uint32_t j = (c0 + w - 1) >> sh; (j << sh) < end; ++j)
                tl[j] = make_uint2(c0 | (f << 16), (uint32_t)((int)s + mn));
        }
        carry += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0 && carry != M) *s_bad = 1;
}

// ------------------------------------------------------------ the decode loop

struct TileCtx {
    int64_t nvec;
    uint32_t V, T, nq;
    uint32_t f0c, f1c, cmin;  // coset table: f of symbol 0, of symbol 1, its min
    uint32_t b;
};

template <typename Lut, int B_CT>
__device__ __forceinline__ uint32_t xshift(uint32_t x, uint32_t b) {
    if constexpr (B_CT > 0) return x >> B_CT;
    else return x >> b;
}

// One renormalisation step for all lanes of the warp.
__device__ __forceinline__ void renorm(uint32_t& x, uint32_t xn, bool act, uint32_t& pbyte, uint32_t lt) {
    const bool need = act && xn < kStateLow;
    const uint32_t bal = __ballot_sync(kFull, need);
    const uint32_t rank = __popc(bal & lt);
    const uint32_t w = lds_u16(pbyte + 2u * rank);
    const uint32_t xr = need ? ((xn << 16) | w) : xn;
    x = act ? xr : x;
    pbyte += 2u * __popc(bal);
}

template <int DT, typename Lut, int B_CT>
__device__ void decode_tiles(const Params& p, const Lut& lut, const TileCtx& tc, uint8_t* smem) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt = lanemask_lt();
    const uint32_t G = gridDim.x;
    const uint32_t M = 1u << tc.b;
    const uint32_t mmask = M - 1;

    Ring rg;
    rg.ring_s = smem_u32(smem + kOffRing + warp * kRingAllocBytes);
    rg.bar_s = smem_u32(smem + kOffBar + warp * 16);
    rg.seq = 0;
    rg.waited = 0;
    rg.timed_out = false;
    if (lane == 0) {
        mbar_init(rg.bar_s, 1);
        mbar_init(rg.bar_s + 8, 1);
        fence_barrier_init();
    }
    __syncwarp();

    const uint32_t total = p.tix[(size_t)kTileWords * tc.T];
    bool corrupt = false;

    for (uint32_t i = warp;; i += kWarps) {
        const uint64_t t64 = (uint64_t)blockIdx.x + (uint64_t)i * G;
        if (t64 >= tc.T) break;
        const uint32_t t = (uint32_t)t64;
        const int64_t v0 = (int64_t)t * tc.V;
        const uint32_t vt = (uint32_t)((tc.nvec - v0) < (int64_t)tc.V ? (tc.nvec - v0) : (int64_t)tc.V);
        const uint32_t* rec = p.tix + (size_t)kTileWords * t;
        const uint32_t off0 = rec[0], off1 = rec[kTileWords];
        uint32_t x = rec[1 + lane];
        const bool bad_rec = !(off0 <= off1 && off1 <= total) || x < kStateLow || x >= 0x80000000u;
        if (__any_sync(kFull, bad_rec)) {
            corrupt = true;
            continue;
        }
        // payload staging bookkeeping (warp-uniform)
        const uint32_t base = off0 & ~7u;
        const uint32_t fend = (off1 + 7u) & ~7u;
        const uint32_t nchunks = (fend - base + kChunkWords - 1) >> kChunkShift;
        const uint32_t seq0 = rg.seq;
        const uint32_t org = (seq0 & 1u) * kChunkWords;
        auto issue = [&](uint32_t ci) {
            const uint32_t w0 = base + ci * kChunkWords;
            const uint32_t n = fend - w0 < (uint32_t)kChunkWords ? fend - w0 : (uint32_t)kChunkWords;
            ring_issue(rg, p.tiles + w0, n, lane);
        };
        if (nchunks > 0) issue(0);
        if (nchunks > 1) issue(1);
        uint32_t cur = off0 - base;  // tile-relative word cursor

        // row of every lane's vector: vector g = v0 + 32r + lane
        const int64_t rowbase = v0 / tc.nq;
        uint32_t ql = (uint32_t)(v0 - rowbase * tc.nq) + lane;
        uint32_t rowl = (uint32_t)rowbase;
        while (ql >= tc.nq) {
            ql -= tc.nq;
            ++rowl;
        }

        const uint32_t rounds = (vt + 31) >> 5;
        for (uint32_t r = 0; r < rounds; ++r) {
            // ---- a3: staging: issue the chunk after the current one, wait for what this round may read
            const uint32_t ci = cur >> kChunkShift;
            if (ci + 1 < nchunks && ci + 1 >= rg.seq - seq0) issue(ci + 1);
            uint32_t last = (cur + kRoundWords - 1) >> kChunkShift;
            const uint32_t issued = rg.seq - seq0;
            if (last >= issued) last = issued - 1;  // never wait on a chunk that was not issued
            while (issued > 0 && rg.waited - seq0 <= last) ring_wait_one(rg);
            uint32_t pbyte = rg.ring_s + 2u * ((org + cur) & (kRingWords - 1));
            const uint32_t p_start = pbyte;

            const uint32_t u = (r << 5) + lane;
            const bool act = u < vt;
            const int64_t g = v0 + u;
            const float sigma = act ? __ldg(p.scales + rowl) : 0.0f;

            // ---- a4: field 0, the coset bit (two-symbol table, no LUT)
            uint32_t slot = x & mmask;
            const uint32_t cs = slot >= tc.f0c ? 1u : 0u;
            {
                const uint32_t f = cs ? tc.f1c : tc.f0c;
                const uint32_t bias = cs ? slot - tc.f0c : slot;
                const uint32_t xn = f * xshift<Lut, B_CT>(x, tc.b) + bias;
                renorm(x, xn, act, pbyte, lt);
            }
            const int c = (int)(tc.cmin + cs);
            const uint32_t cb = lut.coset_base(c & 1);
            bool badsym = false;
            int z[8];
            uint32_t xn;
#define EP_FIELD(K)                                        \
    xn = x;                                                \
    z[K - 1] = lut.template decode<K>(xn, cb, badsym);     \
    renorm(x, xn, act, pbyte, lt);
            EP_FIELD(1)
            EP_FIELD(2)
            EP_FIELD(3)
            EP_FIELD(4)
            EP_FIELD(5)
            EP_FIELD(6)
            EP_FIELD(7)
            EP_FIELD(8)
#undef EP_FIELD
            corrupt |= badsym && act;
            cur += (pbyte - p_start) >> 1;

            // ---- a5: z8 = 2m + parity(z1..z7)
            const int s7 = z[0] + z[1] + z[2] + z[3] + z[4] + z[5] + z[6];
            z[7] = 2 * z[7] + (s7 & 1);

            if (act) {
                if constexpr (DT == EP_LATTICE_I32) {
                    int4* o = reinterpret_cast<int4*>(p.out) + 2 * g;
                    o[0] = make_int4(2 * z[0] + c, 2 * z[1] + c, 2 * z[2] + c, 2 * z[3] + c);
                    o[1] = make_int4(2 * z[4] + c, 2 * z[5] + c, 2 * z[6] + c, 2 * z[7] + c);
                } else {
                    // ---- a6: w = fl32(sigma * (z + c/2)) with one rounding
                    float w[8];
                    if (fabsf(sigma) >= 0x1p-124f) {
                        const float add = c ? sigma * 0.5f : -0.0f;
#pragma unroll
                        for (int k = 0; k < 8; ++k) w[k] = fmaf(sigma, __int2float_rn(z[k]), add);
                    } else {
                        const float hc = c ? 0.5f : 0.0f;
#pragma unroll
                        for (int k = 0; k < 8; ++k) w[k] = sigma * (__int2float_rn(z[k]) + hc);
                    }
                    // ---- a7: conversion + one vector store per lane
                    Out<DT>::store(p.out, g, w);
                }
            }
            // advance every lane's row by 32 vectors
            ql += 32;
            while (ql >= tc.nq) {
                ql -= tc.nq;
                ++rowl;
            }
        }
        // tile end: every lane back at 2^15 and the cursor on the next offset
        const bool lane_ok = x == kStateLow;
        if (!__all_sync(kFull, lane_ok) || cur != off1 - base) corrupt = true;
        // drain the copies of this tile before the ring is reused
        while (rg.waited < rg.seq) ring_wait_one(rg);
        if (rg.timed_out) break;
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

template <int DT>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    int* s_min = reinterpret_cast<int*>(smem + kOffDesc);
    uint32_t* s_A = reinterpret_cast<uint32_t*>(smem + kOffDesc + 128);
    uint32_t* s_off = reinterpret_cast<uint32_t*>(smem + kOffDesc + 256);
    volatile int* s_flag = reinterpret_cast<volatile int*>(smem + kOffFlag);

    // ---- header (every thread reads the same words, so every decision is uniform)
    const uint32_t* h = reinterpret_cast<const uint32_t*>(p.ft);
    const int64_t* h64 = reinterpret_cast<const int64_t*>(p.ft);
    const uint32_t b = h[kHB], V = h[kHV], T = h[kHT];
    const int64_t nvec = p.rows * (p.cols / 8);
    bool ok = h[kHMagic] == kMagic && h[kHVersion] == kVersion && h[kHJ] == (uint32_t)kLanes && b >= (uint32_t)kMinB &&
              b <= (uint32_t)kMaxB && V >= 1 && h64[kHRows64] == p.rows && h64[kHCols64] == p.cols;
    ok = ok && (int64_t)T == (nvec + V - 1) / V;
    const bool unsupported = ok && (h[kHNTab] != (uint32_t)kTables || h[kHFlags] != 0u);
    if (!ok || unsupported) {
        if (threadIdx.x == 0 && blockIdx.x == 0) raise_status(ok ? kStUnsupported : kStHeader);
        return;
    }
    if (blockIdx.x >= T) return;
    const uint32_t M = 1u << b;

    // ---- a2: table descriptors, validation, mode
    if (threadIdx.x < 32) {
        const int t = threadIdx.x;
        int mn = 0;
        uint32_t A = 0;
        if (t < kTables) {
            mn = static_cast<int>(h[12 + 2 * t]);
            A = h[13 + 2 * t];
        }
        const uint32_t incl = warp_incl_scan(A, t);
        if (t < kTables) {
            s_min[t] = mn;
            s_A[t] = A;
            s_off[t] = incl - A;
        }
        bool bad = t < kTables && A > M;
        if (t == 0) bad = bad || A < 1 || A > 2 || mn < 0 || mn + (int)A > 2;
        int packed = 0;
        if (b <= 11) {
            const int64_t zlim = 1ll << (31 - 2 * b);
            const bool fits = t == 0 || t >= kTables || A == 0 || (mn >= -zlim && (int64_t)mn + A - 1 < zlim);
            packed = __all_sync(kFull, fits) ? 1 : 0;
        }
        const bool anybad = __any_sync(kFull, bad);
        if (t == 0) {
            s_flag[0] = anybad ? 1 : 0;
            s_flag[1] = packed ? (int)b : kModeCoarse;
        }
    }
    __syncthreads();
    if (s_flag[0]) {
        if (threadIdx.x == 0) raise_status(kStHeader);
        return;
    }
    const int mode = s_flag[1];
    const uint16_t* fq = reinterpret_cast<const uint16_t*>(p.ft + table_header_bytes(kTables));

    TileCtx tc;
    tc.nvec = nvec;
    tc.V = V;
    tc.T = T;
    tc.nq = (uint32_t)(p.cols / 8);
    tc.b = b;
    tc.cmin = (uint32_t)s_min[0];
    tc.f0c = fq[0];
    tc.f1c = s_A[0] == 2 ? (uint32_t)fq[1] : 0u;
    if (s_A[0] == 1) tc.f0c = M;  // one-symbol coset table: every slot is that symbol
    const bool bad_c = tc.f0c + tc.f1c != M;

    // cooperative LUT build
    switch (mode) {
        case kModePacked9: build_packed<9>(smem, fq, s_min, s_A, s_off, s_flag); break;
        case kModePacked10: build_packed<10>(smem, fq, s_min, s_A, s_off, s_flag); break;
        case kModePacked11: build_packed<11>(smem, fq, s_min, s_A, s_off, s_flag); break;
        default: {
            const uint32_t k = b < (uint32_t)kCoarseBits ? b : (uint32_t)kCoarseBits;
            build_coarse(smem, fq, b, b - k, k, s_min, s_A, s_off, s_flag);
        }
    }
    fence_proxy_async_smem();  // generic writes to the ring area happen before its bulk copies
    __syncthreads();
    if (s_flag[0] || bad_c) {
        if (threadIdx.x == 0) raise_status(kStHeader);
        return;
    }

    switch (mode) {
        case kModePacked9: decode_tiles<DT, PackedLut<9>, 9>(p, PackedLut<9>{smem_u32(smem + kOffLut)}, tc, smem); break;
        case kModePacked10:
            decode_tiles<DT, PackedLut<10>, 10>(p, PackedLut<10>{smem_u32(smem + kOffLut)}, tc, smem);
            break;
        case kModePacked11:
            decode_tiles<DT, PackedLut<11>, 11>(p, PackedLut<11>{smem_u32(smem + kOffLut)}, tc, smem);
            break;
        default: {
            const uint32_t k = b < (uint32_t)kCoarseBits ? b : (uint32_t)kCoarseBits;
            CoarseLut cl;
            cl.lut_s = smem_u32(smem + kOffLut);
            cl.b = b;
            cl.mmask = M - 1;
            cl.sh = b - k;
            cl.nb_shift = k;
            cl.fq = fq;
            cl.s_min = s_min;
            cl.s_A = s_A;
            cl.s_off = s_off;
            decode_tiles<DT, CoarseLut, 0>(p, cl, tc, smem);
        }
    }
}

// ------------------------------------------------------------- host side

int g_num_sms[64];
bool g_attr_done[64][8];
std::mutex g_mu;

template <int DT>
cudaError_t launch(const Params& prm, cudaStream_t st, int dev) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_num_sms[dev]) {
            cudaError_t e = cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
        }
        if (!g_attr_done[dev][DT]) {
            cudaError_t e =
                cudaFuncSetAttribute(decode_kernel<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            if (e != cudaSuccess) return e;
            g_attr_done[dev][DT] = true;
        }
    }
    decode_kernel<DT><<<g_num_sms[dev], kThreads, kSmemBytes, st>>>(prm);
    return cudaGetLastError();
}

}  // namespace
}  // namespace ep

extern "C" {

ep_status ep_decode_tensor(void* stream, const uint16_t* tiles, const uint32_t* tile_index,
                           const uint8_t* freq_tables, const float* row_scales, int64_t rows, int64_t cols,
                           ep_dtype out_dtype, void* out) {
    using namespace ep;
    if (!tiles || !tile_index || !freq_tables || !row_scales || !out) return EP_EINVAL;
    if (rows <= 0 || cols <= 0) return EP_EINVAL;
    if (cols % 8) return EP_EUNSUPPORTED;
    if ((int)out_dtype < EP_BF16 || (int)out_dtype > EP_LATTICE_I32) return EP_EUNSUPPORTED;
    const int64_t nvec = rows * (cols / 8);
    if (nvec >= (1ll << 31) || rows >= (1ll << 31)) return EP_EINVAL;
    auto misaligned = [](const void* q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) != 0; };
    if (misaligned(tiles, 16) || misaligned(freq_tables, 16) || misaligned(tile_index, 4) ||
        misaligned(row_scales, 4) || misaligned(out, 16))
        return EP_EINVAL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EP_ECUDA;
    Params prm{tiles, tile_index, freq_tables, row_scales, out, rows, cols};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    switch (out_dtype) {
        case EP_BF16: e = launch<EP_BF16>(prm, st, dev); break;
        case EP_FP16: e = launch<EP_FP16>(prm, st, dev); break;
        case EP_FP8_E4M3: e = launch<EP_FP8_E4M3>(prm, st, dev); break;
        case EP_INT8: e = launch<EP_INT8>(prm, st, dev); break;
        case EP_FP32: e = launch<EP_FP32>(prm, st, dev); break;
        default: e = launch<EP_LATTICE_I32>(prm, st, dev); break;
    }
    return e == cudaSuccess ? EP_OK : EP_ECUDA;
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
    if (v & (ep::kStHeader | ep::kStCorrupt | ep::kStTimeout)) return EP_ECORRUPT;
    if (v & ep::kStUnsupported) return EP_EUNSUPPORTED;
    return EP_OK;
}

}  // extern "C"

extern "C" const char* ep_status_string(ep_status s) {
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
