// topk_layout.cuh -- tile sizes and workspace layout of the top-k step.
#pragma once

#include <cstdint>

namespace gce {

constexpr int kTkThreads = 256;                    // main pass: 256 threads x 32 elements
constexpr int kTkPerThread = 32;
constexpr int kTkTile = kTkThreads * kTkPerThread;  // 8192 elements per main tile
constexpr int kTkBins = 2048;                      // radix bins per level (11 bits)
constexpr int kTkSampleChunk = 32;                 // sampled run length (one 128-B line)
constexpr int kTkSampleStride = 2048;              // one run per 2048 elements
constexpr int64_t kTkSamplePart = int64_t(1) << 20; // elements covered by one sample unit
constexpr int64_t kTkSampleMinN = 65536;           // smaller layers spill everything
constexpr int kTkHUnit = 8192;                     // spill entries per histogram unit

// Per (worker, layer) state of one top-k step.
struct TkSeg {
    int32_t k;           // 0: layer skipped (k out of range)
    uint32_t lo;         // spill bound: entries with key >= lo are kept as candidates
    int32_t spill_main;  // candidates written by the main pass
    int32_t spill_redo;  // candidates written by the exact fallback pass
    int32_t count;       // candidates used for the selection
    int32_t done_s, done_1, done_2, done_3;  // last-block counters
    uint32_t prefix;     // key bits fixed so far by the radix selection
    int32_t need;        // rank still to find below the prefix; after level 3:
                         // how many entries with key == T are taken
    int32_t pad[5];
};
static_assert(sizeof(TkSeg) == 64, "TkSeg is one 64-byte record");

// The spill entry: the candidate's value and its layer-local index.
struct TkEntry {
    float v;
    int32_t i;
};

}  // namespace gce
