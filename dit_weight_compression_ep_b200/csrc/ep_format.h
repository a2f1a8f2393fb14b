// ep_format.h -- byte layout of the stored representation, as the library reads
// and writes it (see include/entropack.h for the full description).
// EntroPack paper §3.6 "Stored representation"; App. A.3 (17 tables);
// App. C.3 (J = 32 states and a 32-bit offset per tile; states in [2^15, 2^31);
// 16-bit words; b in [9, 15]).
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define EP_HD __host__ __device__
#else
#define EP_HD
#endif

namespace ep {

constexpr uint32_t kMagic = 0x314B5045u;  // "EPK1"
constexpr uint32_t kVersion = 1;
constexpr int kLanes = 32;               // J
constexpr int kFields = 9;               // c, z1..z7, m
constexpr int kTables = 17;              // 1 + 2 x 8
constexpr int kHeaderFixedBytes = 48;
constexpr int kTileWords = 33;           // offset + 32 states
constexpr uint32_t kStateLow = 1u << 15;
constexpr int kMinB = 9, kMaxB = 15;

// header word offsets (u32 units)
constexpr int kHMagic = 0, kHVersion = 1, kHB = 2, kHV = 3, kHJ = 4, kHT = 5;
constexpr int kHRows64 = 3, kHCols64 = 4;  // i64 units
constexpr int kHNTab = 10, kHFlags = 11;

EP_HD inline constexpr int64_t table_header_bytes(int ntab) {
    return (kHeaderFixedBytes + 8 * (int64_t)ntab + 15) / 16 * 16;
}

// table of field k (0 = c, 1..8 = z1..z7, m) for a vector in coset c
EP_HD inline constexpr int table_index(int k, int c) { return k == 0 ? 0 : 1 + 2 * (k - 1) + c; }

}  // namespace ep
