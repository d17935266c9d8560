// topk_layout.cuh -- tile sizes and per-layer state of the top-k step.
#pragma once

#include <cstdint>

namespace gce {

constexpr int kTkThreads = 256;                    // main pass: 256 threads x 32 elements
constexpr int kTkPerThread = 32;
constexpr int kTkTile = kTkThreads * kTkPerThread;  // 8192 elements per main tile
constexpr int kTkBins = 4096;                      // radix bins per level
constexpr int kTkFine = 3072;                      // level-1 bins inside the sampled bracket
constexpr int kTkSBins = 4096;                     // sample bins: 2^19 keys, 16 per octave
constexpr int kTkSampleChunk = 32;                 // sampled run length (one 128-B line)
constexpr int kTkSampleStride = 4096;              // one run per 4096 elements
constexpr int64_t kTkSamplePart = int64_t(1) << 20; // elements covered by one sample unit
constexpr int64_t kTkSampleMinN = 65536;           // smaller layers: exact histogram of all
constexpr int kTkHUnit = 16384;                    // candidates per histogram unit
constexpr int kTkListMax = 65536;                  // longest list of keys in T's level-1 bin

// Per (worker, layer) state of one top-k step.
struct TkSeg {
    int32_t k;           // 0: layer skipped (k out of range)
    uint32_t lo;         // candidates: every element with key >= lo
    uint32_t hi;         // elements with key > hi get memory +0 in the main pass
    int32_t spill_main;  // candidates listed by the main pass
    int32_t spill_redo;  // candidates listed by the exact fallback
    int32_t count;       // candidates used for the selection
    int32_t redo;        // 1: the main list was short; the layer was re-listed whole
    int32_t done_s, done_1, done_2, done_3;  // last-block counters
    uint32_t prefix;     // lowest key of the range that holds T (T once width is 1)
    int32_t need;        // rank of T, counted from the top, inside that range; once
                         // resolved: how many keys equal to T are taken
    uint32_t top;        // T <= top almost surely (sample bound); level 1's fine bins
                         // span [lo, top]
    uint32_t width;      // keys in the range [prefix, prefix + width) that holds T
    int32_t list_mode;   // 1: T is found from a list of the keys in level 1's bin
    int32_t list_n;      // keys appended to that list by the count pass
    int32_t pad[3];
};
static_assert(sizeof(TkSeg) == 80, "TkSeg is one 80-byte record");

}  // namespace gce
