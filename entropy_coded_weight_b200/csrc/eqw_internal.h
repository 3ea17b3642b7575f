// Internal definitions shared by the libeqw translation units (host side).
// Format constants follow container v1 (magic "EQW1"): 12-bit frequencies,
// 32 lanes, 8 consecutive symbols per lane per 256-symbol group, 65536-symbol
// chunks, 256-byte section alignment, 16-byte chunk records.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/eqw.h"

namespace eqw {

constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeaderBytes = 64;
constexpr uint32_t kDirEntryBytes = 64;
constexpr uint32_t kProbBits = 12;
constexpr uint32_t kProbTotal = 1u << kProbBits;
constexpr uint32_t kLanes = 32;
constexpr uint32_t kGroup = 8;
constexpr uint32_t kGroupSyms = kLanes * kGroup;
constexpr uint32_t kChunkSyms = 65536;
constexpr uint32_t kStateLow = 1u << 16;
constexpr uint32_t kRecordHeadBytes = 16 + 4 * kLanes;  // counts + 32 states
constexpr uint64_t kSectionAlign = 256;
constexpr uint32_t kMaxMatsPerLaunch = 16;
constexpr uint32_t kCodecRans = 0;
constexpr uint32_t kCodecHuffman = 1;
constexpr uint32_t kHuffMaxLen = 12;          // longest Huffman code; refill below this many held bits
constexpr uint32_t kHuffRecordHeadBytes = 16; // counts only (no states)

inline uint32_t record_head_bytes(uint32_t codec) {
    return codec == kCodecHuffman ? kHuffRecordHeadBytes : kRecordHeadBytes;
}

inline uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

// A named NVTX range over a host entry point: encode, decode and consumer
// calls show up by name on a profiler's timeline (a no-op when none is attached).
struct NvtxScope {
    explicit NvtxScope(const char *name) { nvtxRangePushA(name); }
    ~NvtxScope() { nvtxRangePop(); }
    NvtxScope(const NvtxScope &) = delete;
    NvtxScope &operator=(const NvtxScope &) = delete;
};

struct MatrixDesc {
    eq_matrix_info info;
    uint64_t chunk_index_off;
    uint64_t scales_off;
    uint64_t outliers_off;
    bool small_scales;    // every scale finite with |scale| < 2^8 (E4M3 single-multiply dequant is exact)
    uint32_t codec;       // kCodecRans or kCodecHuffman
    uint32_t n_present0;  // distinct symbols in the first chunk's table (all chunks' when uniform_table)
};

}  // namespace eqw

struct eq_model {
    const uint8_t *d_blob;
    size_t len;
    uint32_t n_layers;
    uint32_t sm_limit = 0;  // decode launches use at most this many SMs (0: all)
    std::vector<eqw::MatrixDesc> mats;
    std::vector<uint32_t> layer_first;
    std::vector<uint32_t> layer_count;
};
