// latency_probe.cu -- latencies of the operations on the decode step's dependent chain.
//
// One warp runs chains of dependent operations and times each with clock64: the shared
// loads of the lookup table and of the payload ring (App. C.3, "Decoder lookup tables";
// §3.6 one state per lane), the ballot and population counts of the renormalisation, a
// shuffle (the alternative to a shared load for fetching a word), an integer multiply-add
// (state update, addresses) and a warp reduction.  Every operation is emitted from inline
// PTX so that the compiler cannot fold a chain.  Used by `bench.py --latency`; not part of
// the codec.  Built as its own small library (libep_probe.so).
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kChains = 10;
constexpr int kTable = 1024;  // 32-bit words of the shared pointer-chase table (4 KB)

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t imad(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t v;
    asm volatile("mad.lo.u32 %0, %1, %2, %3;" : "=r"(v) : "r"(a), "r"(b), "r"(c));
    return v;
}
__device__ __forceinline__ uint32_t ballot_bit2(uint32_t v) {  // ballot of (v & 4) != 0
    uint32_t b;
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b32 t;\n\tand.b32 t, %1, 4;\n\tsetp.ne.u32 p, t, 0;\n\t"
        "vote.sync.ballot.b32 %0, p, -1;\n\t}"
        : "=r"(b)
        : "r"(v));
    return b;
}
__device__ __forceinline__ uint32_t popc(uint32_t v) {
    uint32_t r;
    asm volatile("popc.b32 %0, %1;" : "=r"(r) : "r"(v));
    return r;
}
__device__ __forceinline__ uint32_t shfl(uint32_t v, uint32_t src) {
    uint32_t r;
    asm volatile("shfl.sync.idx.b32 %0, %1, %2, 31, -1;" : "=r"(r) : "r"(v), "r"(src));
    return r;
}
__device__ __forceinline__ uint32_t redux_add(uint32_t v) {
    uint32_t r;
    asm volatile("redux.sync.add.u32 %0, %1, -1;" : "=r"(r) : "r"(v));
    return r;
}

// chains[k] = clock cycles of n iterations of chain k (lane 0 writes them)
__global__ void probe_kernel(unsigned long long* chains, uint32_t* sink, int n, uint32_t one) {
    __shared__ uint32_t tab[kTable];
    const int lane = threadIdx.x;
    // a pointer chase through a permutation of the table (byte offsets); i -> 17 i + 5 keeps the
    // lanes of every step in distinct banks
    for (int i = lane; i < kTable; i += 32) tab[i] = ((uint32_t)(i * 17 + 5) & (kTable - 1)) * 4u;
    __syncwarp();
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(tab);
    uint32_t lt;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt));
    uint32_t acc = 0;
    int k = 0;
#define EP_CHAIN(BODY)                                       \
    {                                                        \
        uint32_t v = (uint32_t)lane * 4u;                    \
        __syncwarp();                                        \
        const unsigned long long t0 = clock64();             \
        for (int i = 0; i < n; ++i) { BODY; }                \
        const unsigned long long t1 = clock64();             \
        acc += v;                                            \
        if (lane == 0) chains[k] = t1 - t0;                  \
        ++k;                                                 \
    }
    // 0: integer multiply-add (the state update)
    EP_CHAIN(v = imad(v, 3u * one, one))
    // 1: shared 32-bit load, address = base + previous value (one add)
    EP_CHAIN(v = lds32(imad(v, one, base)))
    // 2: shared 16-bit load (the payload word), same address arithmetic
    EP_CHAIN(v = lds16(imad(v, one, base)))
    // 3: ballot of a bit of the value (and + compare + vote), folded back with one multiply-add
    EP_CHAIN(v = imad(ballot_bit2(v), one, v))
    // 4: population count, folded back with one multiply-add
    EP_CHAIN(v = imad(popc(v), one, v))
    // 5: shuffle with the source lane taken from the value (shift + shuffle)
    EP_CHAIN(v = shfl(v, v >> 2))
    // 6: the renormalisation's word index: ballot, and with lanemask_lt, popc, multiply-add
    EP_CHAIN(v = imad(popc(ballot_bit2(v) & lt), 4u * one, v))
    // 7: the same, then the word's shared load (the renormalisation's critical path)
    EP_CHAIN(v = lds16(imad(popc(ballot_bit2(v) & lt), 4u * one, base)))
    // 8: the same with a shuffle in place of the address arithmetic and the shared load
    EP_CHAIN(v = shfl(v, popc(ballot_bit2(v) & lt)) + 4u)
    // 9: warp reduction (redux.sync.add), folded back with one multiply-add
    EP_CHAIN(v = imad(redux_add(v), one, v))
#undef EP_CHAIN
    sink[lane] = acc;
}

}  // namespace

// Run the probe once on the current device (one warp) and write the cycles per iteration of
// each chain to cycles_per_op[0 .. min(n_out, 10)).  Returns 0, or the CUDA error code.
extern "C" int ep_probe_latencies(double* cycles_per_op, int n_out) {
    unsigned long long* d = nullptr;
    uint32_t* s = nullptr;
    const int n = 4096;
    cudaError_t e = cudaMalloc(&d, kChains * sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMalloc(&s, 32 * sizeof(uint32_t));
    unsigned long long h[kChains] = {};
    for (int rep = 0; rep < 3 && e == cudaSuccess; ++rep) {  // the last of three runs (warm caches)
        probe_kernel<<<1, 32>>>(d, s, n, 1u);
        e = cudaDeviceSynchronize();
        if (e == cudaSuccess) e = cudaMemcpy(h, d, sizeof(h), cudaMemcpyDeviceToHost);
    }
    if (d) cudaFree(d);
    if (s) cudaFree(s);
    if (e != cudaSuccess) return (int)e;
    for (int k = 0; k < kChains && k < n_out; ++k) cycles_per_op[k] = (double)h[k] / n;
    return 0;
}
