// randk.cu -- Mem-SGD error-feedback rand-k step on sm_100a.
//
// "Sparsified SGD with Memory", Method / Abstract: the same error-feedback
// update as top-k with comp_k keeping k random coordinates, values unscaled.
// The k coordinates are the k smallest (key, index) pairs, key_i = the high
// 32 bits of output i+1 of a SplitMix64 generator (Steele, Lea, Flood 2014)
// whose state is derived from (seed, stream 0, worker, layer, step).
//
// The choice does not depend on the data, so it is made before the memory
// pass, without touching HBM:
//   keys     hash every index once: a bitmask of key < lo (1 bit / element),
//            the count below lo per tile, and a short list of the keys in
//            [lo, hi] -- a band of +-sigma binomial deviations around the
//            expected k-th smallest key
//   resolve  exact (key, index) selection inside the band (one CTA per
//            layer); the chosen band entries are OR-ed into the bitmask
//   keys/resolve again with the band opened to everything for any layer
//            whose band missed (exact fallback; results never depend on sigma)
//   scan     per-tile output offsets
//   emit     the only HBM pass: v = fl(m + fl(eta*g)), ordered write of the
//            chosen (v, i), mem <- v or +0; with the look-ahead, a third of
//            each block's warps hash the next step's keys meanwhile
// DRAM traffic: 12 B per element + 8 B per chosen entry + 1/8 B of bitmask
// written and read.
#include <cmath>

#include "common.cuh"
#include "scan.cuh"
#include "topk_layout.cuh"

namespace gce {



struct RkSeg {
    int32_t k;       // 0: layer skipped
    uint32_t lo, hi; // band of candidate keys
    int32_t c_lo;    // keys below lo (main pass)
    int32_t cand;    // band entries listed (main pass)
    int32_t cand_redo;
    int32_t fail;    // 1: the band missed the k-th key; redone exactly
    uint32_t T;      // chosen iff key < T or (key == T and i <= iT)
    int32_t iT;
    uint64_t base;   // hash state of this (worker, layer, step)
    int32_t pad[3];
};
static_assert(sizeof(RkSeg) == 56 || sizeof(RkSeg) == 64, "RkSeg layout");

struct RkEntry {
    uint32_t key;
    int32_t i;
};

constexpr int kRkWords = kTkTile / 32;  // bitmask words per tile (256)

struct RkLayout {
    int64_t S = 0, TT = 0;
    size_t segs = 0, tile_cnt = 0, bitmask = 0, cand = 0, total = 0;
};

// Threads of the look-ahead emit block: kTkThreads stream the memory, the
// other kRkHashThreads hash the next step's keys.
constexpr int kRkHashThreads = 128;
constexpr int kRkSplitThreads = kTkThreads + kRkHashThreads;

static RkLayout rk_layout(const gce_table* t, int32_t W) {
    RkLayout o;
    Carver c;
    const bool on = t->ckind == GCE_KIND_RANDK;
    o.S = on ? int64_t(W) * int64_t(t->comp.size()) : 0;
    o.TT = on ? int64_t(W) * t->tiles_pw : 0;
    // two sets of each, by step parity: this step's and the next one's
    o.segs = c.take<RkSeg>(2 * o.S);
    o.tile_cnt = c.take<int32_t>(2 * o.TT);
    o.bitmask = c.take<uint32_t>(2 * o.TT * kRkWords);
    o.cand = c.take<RkEntry>(o.S ? int64_t(W) * t->comp_N : 0);
    o.total = c.off;
    return o;
}

size_t randk_ws_bytes(const gce_table* t, int32_t W) { return rk_layout(t, W).total; }

// State of (worker, layer) segment s for `step`: k (0 when out of range),
// the band [lo, hi] of +-(sigma * binomial sd + sigma) keys around the
// expected k-th smallest key, the generator state, counters at zero.  The
// generator takes the job-wide worker index worker0 + s / ncomp.
__device__ __forceinline__ void rk_setup_seg(int64_t s, const DevLayer* __restrict__ layers,
                                             const int32_t* __restrict__ comp, int32_t ncomp,
                                             const int32_t* __restrict__ k_or_rank, uint64_t seed,
                                             uint64_t worker0, uint64_t step, double sigma,
                                             RkSeg* __restrict__ segs,
                                             int32_t* __restrict__ status) {
    const int32_t l = comp[s % ncomp];
    const DevLayer L = layers[l];
    const int32_t k = k_or_rank ? k_or_rank[l] : L.cap;
    RkSeg g{};
    if (k >= 1 && k <= L.cap && int64_t(k) <= L.n) {
        g.k = k;
    } else {
        g.k = 0;
        if (status) set_status(status, GCE_STATUS_K_RANGE);
    }
    const double n = double(L.n), p = double(k) / n;
    const double d = sigma * (sqrt(n * p * (1.0 - p)) + 1.0);
    const double scale = 4294967296.0 / n;
    const double lo = (double(k) - d) * scale, hi = (double(k) + d) * scale;
    g.lo = lo <= 0.0 ? 0u : (lo >= 4294967295.0 ? 0xFFFFFFFFu : uint32_t(lo));
    g.hi = hi >= 4294967295.0 ? 0xFFFFFFFFu : (hi <= 0.0 ? 0u : uint32_t(hi));
    if (g.hi < g.lo) g.hi = g.lo;
    g.base = hash_base(seed, 0, worker0 + uint64_t(s / ncomp), uint64_t(l), step);
    segs[s] = g;
}

// tag: where the workspace records which step's key pass it holds; block 0
// writes tag_value there (0: none).
__global__ void __launch_bounds__(256) rk_setup_kernel(const DevLayer* __restrict__ layers,
                                                       const int32_t* __restrict__ comp,
                                                       int32_t ncomp, int64_t S,
                                                       const int32_t* __restrict__ k_or_rank,
                                                       uint64_t seed, uint64_t worker0,
                                                       uint64_t step, double sigma,
                                                       RkSeg* __restrict__ segs,
                                                       int32_t* __restrict__ status,
                                                       uint64_t* __restrict__ tag,
                                                       uint64_t tag_value) {
    grid_dependency_sync();
    if (blockIdx.x == 0 && threadIdx.x == 0) *tag = tag_value;
    for (int64_t s = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; s < S;
         s += int64_t(gridDim.x) * blockDim.x)
        rk_setup_seg(s, layers, comp, ncomp, k_or_rank, seed, worker0, step, sigma, segs,
                     status);
}

// Barrier over the block (kId 0) or, with a named barrier, over the kThreads
// threads of one warp group.
template <int kId, int kThreads>
__device__ __forceinline__ void group_sync() {
    if constexpr (kId == 0) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"r"(kId), "r"(kThreads) : "memory");
}

// Key pass over one tile t (worker w, layer L): the bitmask words of key < lo,
// the tile's count below lo and the band entries [lo, hi] appended to the
// layer's list.  kRedo: re-list a failed layer whole (band = every key,
// nothing below it).  Run by a group of kThreads threads (gtid = the thread's
// index in it) that syncs on barrier kBar; g.k != 0.
template <bool kRedo, int kThreads = kTkThreads, int kBar = 0>
__device__ __forceinline__ void rk_keys_tile(int64_t t, int w, int lt, const DevLayer& L,
                                             RkSeg& g, int64_t comp_N, int32_t* tile_cnt,
                                             uint32_t* bitmask, RkEntry* cand, int* s_red,
                                             int gtid) {
    constexpr int kChunks = kRkWords / kThreads;  // 32-element words a thread
    static_assert(kChunks * kThreads == kRkWords, "a tile's words split evenly");
    const int lane = gtid & 31, gwarp = gtid >> 5;
    const uint32_t lo = kRedo ? 0u : g.lo, hi = kRedo ? 0xFFFFFFFFu : g.hi;
    const uint32_t span = hi - lo;  // lo <= key <= hi  iff  key - lo <= hi - lo (unsigned)
    const uint64_t base = g.base;
    const int64_t tstart = int64_t(lt - L.tile0) * kTkTile;
    int nbelow = 0;
#pragma unroll 1
    for (int c = 0; c < kChunks; ++c) {
        const int word = gtid + c * kThreads;
        const int64_t e0 = tstart + int64_t(word) * 32;
        const uint64_t x0 = base + uint64_t(e0 + 1) * kGamma;  // generator state of element e0
        uint32_t below = 0, inband = 0;
        if (e0 + 32 <= L.n) {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const uint32_t key = mix64_hi(x0 + uint64_t(q) * kGamma);
                below |= uint32_t(!kRedo && key < lo) << q;  // the redo lists every key
                inband |= uint32_t(key - lo <= span) << q;
            }
        } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const uint32_t key = mix64_hi(x0 + uint64_t(q) * kGamma);
                if (e0 + q < L.n) {
                    below |= uint32_t(!kRedo && key < lo) << q;  // the redo lists every key
                    inband |= uint32_t(key - lo <= span) << q;
                }
            }
        }
        bitmask[t * kRkWords + word] = below;
        nbelow += __popc(below);
        // band entries: order does not matter, the resolve sorts them out
        const int nb = __popc(inband);
        const int incl = warp_inclusive_scan(nb);
        int wbase = 0;
        if (lane == 31 && incl) wbase = atomicAdd(kRedo ? &g.cand_redo : &g.cand, incl);
        wbase = __shfl_sync(kFull, wbase, 31);
        RkEntry* out = cand + int64_t(w) * comp_N + L.sp_off + wbase + (incl - nb);
        int pos = 0;
        while (inband) {  // few band entries: their keys are recomputed
            const int q = __ffs(inband) - 1;
            inband &= inband - 1;
            const uint32_t key = mix64_hi(x0 + uint64_t(q) * kGamma);
            out[pos++] = RkEntry{key, int32_t(e0 + q)};
        }
    }
    // tile count of keys below the band
    const int cw = warp_sum(nbelow);
    if (lane == 0) s_red[gwarp] = cw;
    group_sync<kBar, kThreads>();
    if (gtid == 0) {
        int tot = 0;
        for (int i = 0; i < kThreads / 32; ++i) tot += s_red[i];
        tile_cnt[t] = tot;
        if (tot) atomicAdd(&g.c_lo, tot);
    }
    group_sync<kBar, kThreads>();  // s_red is read before the next tile writes it
}

template <bool kRedo>
__global__ void __launch_bounds__(256) rk_keys_kernel(const DevLayer* __restrict__ layers,
                                                      const int32_t* __restrict__ tile_layer,
                                                      int32_t tiles_pw, int32_t W, int32_t ncomp,
                                                      int64_t comp_N, RkSeg* __restrict__ segs,
                                                      int32_t* __restrict__ tile_cnt,
                                                      uint32_t* __restrict__ bitmask,
                                                      RkEntry* __restrict__ cand) {
    grid_dependency_sync();
    __shared__ int s_red[8];
    const int64_t total = int64_t(tiles_pw) * W;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
        const int w = int(t / tiles_pw);
        const int lt = int(t % tiles_pw);
        const DevLayer L = layers[tile_layer[lt]];
        RkSeg& g = segs[int64_t(w) * ncomp + L.sidx];
        if (g.k == 0) continue;
        if (kRedo && !g.fail) continue;
        rk_keys_tile<kRedo>(t, w, lt, L, g, comp_N, tile_cnt, bitmask, cand, s_red, threadIdx.x);
    }
}

// The k of every (worker, layer) read again for this step (the key pass run
// ahead used the k of the step before, which only sized its band: a band
// that misses the new k-th key sends the layer to the exact fallback).  If
// the workspace does not hold the expected step's key pass (its tag
// differs), every segment is set up afresh and sent to the exact fallback.
__global__ void __launch_bounds__(256) rk_refresh_k_kernel(const DevLayer* __restrict__ layers,
                                                           const int32_t* __restrict__ comp,
                                                           int32_t ncomp, int64_t S,
                                                           const int32_t* __restrict__ k_or_rank,
                                                           uint64_t seed, uint64_t worker0,
                                                           uint64_t step,
                                                           double sigma, RkSeg* __restrict__ segs,
                                                           int32_t* __restrict__ status,
                                                           const uint64_t* __restrict__ tag,
                                                           uint64_t tag_value) {
    grid_dependency_sync();
    const bool held = *tag == tag_value;
    for (int64_t s = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; s < S;
         s += int64_t(gridDim.x) * blockDim.x) {
        if (!held) {
            rk_setup_seg(s, layers, comp, ncomp, k_or_rank, seed, worker0, step, sigma, segs,
                         status);
            segs[s].fail = 1;
            continue;
        }
        const int32_t l = comp[s % ncomp];
        const DevLayer L = layers[l];
        const int32_t k = k_or_rank ? k_or_rank[l] : L.cap;
        if (k >= 1 && k <= L.cap && int64_t(k) <= L.n) {
            segs[s].k = k;
        } else {
            segs[s].k = 0;
            set_status(status, GCE_STATUS_K_RANGE);
        }
    }
}

// One CTA: the rank-th smallest (key, index) pair (rank 1-based) of a list.
__device__ void cta_select_pair(const RkEntry* __restrict__ list, int32_t count, int32_t rank,
                                int32_t* h, uint32_t* s_pref, int32_t* s_rank, uint32_t* T,
                                int32_t* iT) {
    const int tid = threadIdx.x;
    if (tid == 0) {
        *s_pref = 0;
        *s_rank = rank;
    }
    __syncthreads();
    // key bits 31..21, 20..10, 9..0
    const int kshift[3] = {21, 10, 0}, kbits[3] = {11, 11, 10};
    for (int lv = 0; lv < 3; ++lv) {
        const int nb = 1 << kbits[lv], sh = kshift[lv], top = sh + kbits[lv];
        for (int b = tid; b < nb; b += blockDim.x) h[b] = 0;
        __syncthreads();
        const uint32_t pref = *s_pref;
        for (int32_t j = tid; j < count; j += blockDim.x) {
            const uint32_t key = list[j].key;
            if (top >= 32 || (key >> top) == (pref >> top)) atomicAdd(&h[(key >> sh) & (nb - 1)], 1);
        }
        __syncthreads();
        if (tid < 32) {
            int64_t below = 0;
            const int b = warp_find_from_bottom(h, nb, *s_rank, &below);
            if (tid == 0) {
                *s_pref = pref | (uint32_t(max(b, 0)) << sh);
                *s_rank = *s_rank - int32_t(below);
            }
        }
        __syncthreads();
    }
    const uint32_t key_T = *s_pref;
    __syncthreads();  // every thread has read key_T before the prefix is reset
    if (tid == 0) *s_pref = 0;
    __syncthreads();
    // among keys == T: index bits 30..20, 19..9, 8..0
    const int ishift[3] = {20, 9, 0}, ibits[3] = {11, 11, 9};
    for (int lv = 0; lv < 3; ++lv) {
        const int nb = 1 << ibits[lv], sh = ishift[lv], top = sh + ibits[lv];
        for (int b = tid; b < nb; b += blockDim.x) h[b] = 0;
        __syncthreads();
        const uint32_t pref = *s_pref;
        for (int32_t j = tid; j < count; j += blockDim.x) {
            const RkEntry e = list[j];
            const uint32_t i = uint32_t(e.i);
            if (e.key == key_T && (i >> top) == (pref >> top)) atomicAdd(&h[(i >> sh) & (nb - 1)], 1);
        }
        __syncthreads();
        if (tid < 32) {
            int64_t below = 0;
            const int b = warp_find_from_bottom(h, nb, *s_rank, &below);
            if (tid == 0) {
                *s_pref = pref | (uint32_t(max(b, 0)) << sh);
                *s_rank = *s_rank - int32_t(below);
            }
        }
        __syncthreads();
    }
    *T = key_T;
    *iT = int32_t(*s_pref);
    __syncthreads();
}

// One CTA per layer: find (T, iT), then OR the chosen band entries into the
// bitmask and add them to their tiles' counts.
template <bool kRedo>
__global__ void __launch_bounds__(1024) rk_resolve_kernel(const DevLayer* __restrict__ layers,
                                                          const int32_t* __restrict__ comp,
                                                          int32_t ncomp, int64_t S,
                                                          int32_t tiles_pw, int64_t comp_N,
                                                          RkSeg* __restrict__ segs,
                                                          int32_t* __restrict__ tile_cnt,
                                                          uint32_t* __restrict__ bitmask,
                                                          const RkEntry* __restrict__ cand,
                                                          int32_t* __restrict__ status) {
    grid_dependency_sync();
    __shared__ int32_t h[2048];
    __shared__ uint32_t s_pref;
    __shared__ int32_t s_rank;
    __shared__ int s_go;
    for (int64_t s = blockIdx.x; s < S; s += gridDim.x) {
        RkSeg& g = segs[s];
        if (threadIdx.x == 0) {
            int go = 0;
            if (g.k > 0) {
                if (!kRedo) {
                    const int32_t need = g.k - g.c_lo;
                    go = (need >= 1 && need <= g.cand);
                    if (!go) {
                        g.fail = 1;
                        set_status(status, GCE_STATUS_FALLBACK);
                    }
                } else {
                    go = g.fail;
                }
            }
            s_go = go;
        }
        __syncthreads();
        if (!s_go) {
            __syncthreads();
            continue;
        }
        const int w = int(s / ncomp);
        const DevLayer L = layers[comp[s % ncomp]];
        const RkEntry* list = cand + int64_t(w) * comp_N + L.sp_off;
        const int32_t count = kRedo ? g.cand_redo : g.cand;
        const int32_t rank = kRedo ? g.k : g.k - g.c_lo;
        uint32_t T;
        int32_t iT;
        cta_select_pair(list, count, rank, h, &s_pref, &s_rank, &T, &iT);
        if (threadIdx.x == 0) {
            g.T = T;
            g.iT = iT;
        }
        const int64_t t0 = int64_t(w) * tiles_pw + L.tile0;
        for (int32_t j = threadIdx.x; j < count; j += blockDim.x) {
            const RkEntry e = list[j];
            if (e.key < T || (e.key == T && e.i <= iT)) {
                const int64_t t = t0 + e.i / kTkTile;
                const int r = e.i % kTkTile;
                atomicOr(&bitmask[t * kRkWords + r / 32], 1u << (r % 32));
                atomicAdd(&tile_cnt[t], 1);
            }
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(1024) rk_scan_kernel(const DevLayer* __restrict__ layers,
                                                       const int32_t* __restrict__ comp,
                                                       int32_t ncomp, int64_t S, int32_t tiles_pw,
                                                       const RkSeg* __restrict__ segs,
                                                       int32_t* __restrict__ tile_cnt) {
    grid_dependency_sync();
    __shared__ int s_warp[33];
    for (int64_t s = blockIdx.x; s < S; s += gridDim.x) {
        if (segs[s].k == 0) continue;
        const int w = int(s / ncomp);
        const DevLayer L = layers[comp[s % ncomp]];
        int32_t* tc = tile_cnt + int64_t(w) * tiles_pw + L.tile0;
        int carry = 0;
        for (int b0 = 0; b0 < L.ntiles; b0 += blockDim.x) {
            const int i = b0 + threadIdx.x;
            const int x = i < L.ntiles ? tc[i] : 0;
            int tot = 0;
            const int ex = block_exclusive_scan(x, s_warp, &tot);
            if (i < L.ntiles) tc[i] = carry + ex;
            carry += tot;
        }
    }
}

// kNext: the block's first kTkThreads threads run the memory pass (named
// barrier 1) while its last kRkHashThreads threads run the next step's key
// pass (segs_next) over the same tiles into the other parity's bitmask and
// tile counts (named barrier 2): the two groups share no data, so the hash's
// ALU work and the memory traffic overlap on every SM.  Without kNext the
// block is the memory group alone.
template <bool kNext>
__global__ void __launch_bounds__(kNext ? kRkSplitThreads : kTkThreads, kNext ? 2 : 4)
rk_emit_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t W, int32_t ncomp, int64_t N, int64_t vals_pw, int64_t comp_N,
    const float* __restrict__ grad, float* __restrict__ mem, float eta,
    const RkSeg* __restrict__ segs, RkSeg* __restrict__ segs_next, const int32_t* tile_off,
    const uint32_t* bitmask, int32_t* tile_cnt_next, uint32_t* bitmask_next,
    RkEntry* __restrict__ cand, float* __restrict__ vals, int32_t* __restrict__ idx,
    int32_t* __restrict__ status) {
    grid_dependency_sync();
    constexpr int kIters = kTkPerThread / 4;
    constexpr int kWarps = kTkThreads / 32;
    constexpr int kMemBar = kNext ? 1 : 0;
    __shared__ int32_t s_wt[kIters * kWarps];
    __shared__ int s_red[kRkHashThreads / 32];
    __shared__ int32_t s_toff;  // this tile's first payload slot
    const int64_t total = int64_t(tiles_pw) * W;
    if (kNext && threadIdx.x >= kTkThreads) {
        // the hash group
        const int gtid = int(threadIdx.x) - kTkThreads;
        for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
            const int w = int(t / tiles_pw);
            const int lt = int(t % tiles_pw);
            const DevLayer L = layers[tile_layer[lt]];
            RkSeg& gn = segs_next[int64_t(w) * ncomp + L.sidx];
            if (gn.k == 0) continue;
            rk_keys_tile<false, kRkHashThreads, 2>(t, w, lt, L, gn, comp_N, tile_cnt_next,
                                                   bitmask_next, cand, s_red, gtid);
        }
        return;
    }
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
        const int w = int(t / tiles_pw);
        const int lt = int(t % tiles_pw);
        const DevLayer L = layers[tile_layer[lt]];
        // the bulk-copy engine pulls this block's next tile into L2 meanwhile
        if (tid == 0 && t + gridDim.x < total) {
            const int64_t t2 = t + gridDim.x;
            const int lt2 = int(t2 % tiles_pw);
            const DevLayer L2 = layers[tile_layer[lt2]];
            const int64_t s2 = int64_t(lt2 - L2.tile0) * kTkTile;
            const int64_t e2 = int64_t(t2 / tiles_pw) * N + L2.offset + s2;
            if (s2 + kTkTile <= L2.n && (e2 & 3) == 0) {
                prefetch_l2_bulk(grad + e2, kTkTile * 4);
                prefetch_l2_bulk(mem + e2, kTkTile * 4);
            }
            prefetch_l2_bulk(bitmask + t2 * kRkWords, kRkWords * 4);
        }
        const int64_t s = int64_t(w) * ncomp + L.sidx;
        const int32_t k = segs[s].k;
        if (k == 0) continue;
        const int64_t tstart = int64_t(lt - L.tile0) * kTkTile;
        const int cnt = int(min64(kTkTile, L.n - tstart));
        const int64_t ebase = int64_t(w) * N + L.offset + tstart;
        const float* g = grad + ebase;
        float* m = mem + ebase;
        const uint32_t* bm = bitmask + t * kRkWords;
        const bool vec = cnt == kTkTile && (ebase & 3) == 0;
        {
            // every load of the tile issued up front, then the arithmetic; the
            // memory first receives v everywhere, and the few chosen entries
            // are read back and zeroed once their payload slots are known
            uint32_t words[kIters];
#pragma unroll
            for (int j = 0; j < kIters; ++j)
                words[j] = __ldcg(bm + ((j * (kTkThreads * 4) + tid * 4) >> 5));
            if (tid == 0) s_toff = tile_off[t];
            if (vec) {
                float4 gv[kIters], mv[kIters];
#pragma unroll
                for (int j = 0; j < kIters; ++j) {
                    const int e = j * (kTkThreads * 4) + tid * 4;
                    gv[j] = ld_stream4(g + e);
                    mv[j] = ld_stream4(m + e);
                }
                bool bad = false;
#pragma unroll
                for (int j = 0; j < kIters; ++j) {
                    const int e = j * (kTkThreads * 4) + tid * 4;
                    float4 x;
                    x.x = residual(mv[j].x, eta, gv[j].x);
                    x.y = residual(mv[j].y, eta, gv[j].y);
                    x.z = residual(mv[j].z, eta, gv[j].z);
                    x.w = residual(mv[j].w, eta, gv[j].w);
                    bad |= (abs_key(x.x) >= kNonFiniteKey) | (abs_key(x.y) >= kNonFiniteKey) |
                           (abs_key(x.z) >= kNonFiniteKey) | (abs_key(x.w) >= kNonFiniteKey);
                    __stcs(reinterpret_cast<float4*>(m + e), x);
                }
                flag_nonfinite(bad, status);
            } else {
                bool bad = false;
#pragma unroll
                for (int j = 0; j < kIters; ++j) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int e = j * (kTkThreads * 4) + tid * 4 + q;
                        if (e < cnt) {
                            const float x = residual(m[e], eta, __ldcs(g + e));
                            bad |= abs_key(x) >= kNonFiniteKey;
                            m[e] = x;
                        }
                    }
                }
                flag_nonfinite(bad, status);
            }
            uint32_t flags = 0;
#pragma unroll
            for (int j = 0; j < kIters; ++j) {
                const int e = j * (kTkThreads * 4) + tid * 4;
                flags |= ((words[j] >> (e & 31)) & 0xFu) << (4 * j);
            }
            int incl[kIters];
#pragma unroll
            for (int j = 0; j < kIters; ++j) {
                incl[j] = warp_inclusive_scan(__popc((flags >> (4 * j)) & 0xFu));
                if (lane == 31) s_wt[j * kWarps + warp] = incl[j];
            }
            group_sync<kMemBar, kTkThreads>();
            if (warp == 0) {
                const int a = s_wt[2 * lane], b = s_wt[2 * lane + 1];
                const int x = warp_inclusive_scan(a + b);
                s_wt[2 * lane] = x - a - b;
                s_wt[2 * lane + 1] = x - b;
            }
            group_sync<kMemBar, kTkThreads>();
            const int base = s_toff;
            float* vout = vals + int64_t(w) * vals_pw + L.val_off;
            int32_t* iout = idx + int64_t(w) * vals_pw + L.val_off;
#pragma unroll
            for (int j = 0; j < kIters; ++j) {
                const uint32_t f = (flags >> (4 * j)) & 0xFu;
                int pos = base + s_wt[j * kWarps + warp] + incl[j] - __popc(f);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if ((f & (1u << q)) && pos < k) {
                        const int e = j * (kTkThreads * 4) + tid * 4 + q;
                        vout[pos] = m[e];
                        iout[pos] = int32_t(tstart + e);
                        m[e] = 0.0f;
                    }
                    pos += (f >> q) & 1u;
                }
            }
            group_sync<kMemBar, kTkThreads>();  // s_wt and s_toff are consumed
        }
    }
}

}  // namespace gce

using namespace gce;

static int randk_step(const gce_table* t, int32_t W, int64_t worker0, const float* grad,
                      float* mem, float eta, const int32_t* k_or_rank, uint64_t seed,
                      uint64_t step, float* vals, int32_t* idx, void* ws, size_t ws_bytes,
                      void* stream) {
    if (!t || W < 1 || worker0 < 0 || !grad || !mem || !ws) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_RANDK && t->ckind != -1) return GCE_ERR_KIND;
    if (!aligned16(grad) || !aligned16(mem) || !aligned16(ws)) return GCE_ERR_ARG;
    if ((t->vals_pw > 0) && (!vals || !aligned16(vals))) return GCE_ERR_ARG;
    if (t->ckind == GCE_KIND_RANDK && (!idx || !aligned16(idx))) return GCE_ERR_ARG;
    if (k_or_rank && (reinterpret_cast<uintptr_t>(k_or_rank) & 3)) return GCE_ERR_ARG;
    const RkLayout lay = rk_layout(t, W);
    if (ws_bytes < lay.total) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = static_cast<int32_t*>(ws);
    if (lay.S > 0) {
        const int32_t ncomp = int32_t(t->comp.size());
        // this step's bitmask and tile counts, and the next step's (which the
        // look-ahead fills), by step parity
        int32_t* tile_cnt = at<int32_t>(ws, lay.tile_cnt) + (step & 1) * lay.TT;
        uint32_t* bitmask = at<uint32_t>(ws, lay.bitmask) + (step & 1) * lay.TT * kRkWords;
        int32_t* tile_cnt_next = at<int32_t>(ws, lay.tile_cnt) + ((step + 1) & 1) * lay.TT;
        uint32_t* bitmask_next =
            at<uint32_t>(ws, lay.bitmask) + ((step + 1) & 1) * lay.TT * kRkWords;
        RkEntry* cand = at<RkEntry>(ws, lay.cand);
        // Run the next step's key pass inside this step's memory pass unless
        // the stream is being captured (a graph would replay one step number).
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return GCE_ERR_CUDA;
        const double sigma = option_of(t, GCE_OPT_BRACKET_SIGMA);
        const bool pipe = option_of(t, GCE_OPT_RANDK_AHEAD) != 0.0 &&
                          cs == cudaStreamCaptureStatusNone &&
                          step != ~uint64_t(0);
        bool have = false;
        {
            std::lock_guard<std::mutex> lk(t->rk_mu);
            have = pipe && t->rk_valid && t->rk_ws == ws && t->rk_seed == seed &&
                   t->rk_step == step && t->rk_W == W && t->rk_worker0 == worker0;
            t->rk_valid = false;
        }
        // which step's key pass the workspace holds (header bytes 64-71)
        uint64_t* tag = at<uint64_t>(ws, 64);
        auto tag_of = [&](uint64_t sv) {
            const uint64_t h = mix64(mix64(mix64(mix64(seed + kGamma) + sv) + uint64_t(W)) +
                                     uint64_t(worker0)) ^
                               reinterpret_cast<uintptr_t>(t);
            return h ? h : 1u;
        };
        RkSeg* segs = at<RkSeg>(ws, lay.segs) + (step & 1) * lay.S;
        RkSeg* segs_next = at<RkSeg>(ws, lay.segs) + ((step + 1) & 1) * lay.S;
        static const int r_setup = resident_blocks(rk_setup_kernel, 256);
        static const int r_refresh = resident_blocks(rk_refresh_k_kernel, 256);
        static const int r_keys0 = resident_blocks(rk_keys_kernel<false>, 256);
        static const int r_keys1 = resident_blocks(rk_keys_kernel<true>, 256);
        static const int r_res0 = resident_blocks(rk_resolve_kernel<false>, 1024);
        static const int r_res1 = resident_blocks(rk_resolve_kernel<true>, 1024);
        static const int r_scan = resident_blocks(rk_scan_kernel, 1024);
        static const int r_emit0 = resident_blocks(rk_emit_kernel<false>, kTkThreads);
        static const int r_emit1 = resident_blocks(rk_emit_kernel<true>, kRkSplitThreads);
        if (have) {
            GCE_LAUNCH(rk_refresh_k_kernel, wave_grid((lay.S + 255) / 256, 4, r_refresh), 256, 0,
                       st, t->d_layers, t->d_comp, ncomp, lay.S, k_or_rank, seed,
                       uint64_t(worker0), step, sigma, segs, status, tag,
                       tag_of(step));
        } else {
            GCE_LAUNCH(rk_setup_kernel, wave_grid((lay.S + 255) / 256, 4, r_setup), 256, 0, st,
                       t->d_layers, t->d_comp, ncomp, lay.S, k_or_rank, seed,
                       uint64_t(worker0), step, sigma, segs, status, tag,
                       uint64_t(0));
            GCE_LAUNCH(rk_keys_kernel<false>, wave_grid(lay.TT, 8, r_keys0), 256, 0, st,
                       t->d_layers, t->d_tile_layer, t->tiles_pw, W, ncomp, t->comp_N, segs,
                       tile_cnt, bitmask, cand);
        }
        GCE_LAUNCH(rk_resolve_kernel<false>, wave_grid(lay.S, 2, r_res0), 1024, 0, st, t->d_layers,
                   t->d_comp, ncomp, lay.S, t->tiles_pw, t->comp_N, segs, tile_cnt, bitmask, cand,
                   status);
        GCE_LAUNCH(rk_keys_kernel<true>, wave_grid(lay.TT, 8, r_keys1), 256, 0, st, t->d_layers,
                   t->d_tile_layer, t->tiles_pw, W, ncomp, t->comp_N, segs, tile_cnt, bitmask,
                   cand);
        GCE_LAUNCH(rk_resolve_kernel<true>, wave_grid(lay.S, 2, r_res1), 1024, 0, st, t->d_layers,
                   t->d_comp, ncomp, lay.S, t->tiles_pw, t->comp_N, segs, tile_cnt, bitmask, cand,
                   status);
        GCE_LAUNCH(rk_scan_kernel, wave_grid(lay.S, 2, r_scan), 1024, 0, st, t->d_layers, t->d_comp,
                   ncomp, lay.S, t->tiles_pw, segs, tile_cnt);
        if (pipe) {
            // the next step's band from this step's k (a guess: the exact
            // resolve of that step re-reads k and repairs any miss)
            GCE_LAUNCH(rk_setup_kernel, wave_grid((lay.S + 255) / 256, 4, r_setup), 256, 0, st,
                       t->d_layers, t->d_comp, ncomp, lay.S, k_or_rank, seed,
                       uint64_t(worker0), step + 1, sigma, segs_next, nullptr, tag,
                       tag_of(step + 1));
            GCE_LAUNCH(rk_emit_kernel<true>, wave_grid(lay.TT, r_emit1, r_emit1), kRkSplitThreads,
                       0, st, t->d_layers, t->d_tile_layer, t->tiles_pw, W, ncomp, t->N,
                       t->vals_pw, t->comp_N, grad, mem, eta, segs, segs_next, tile_cnt, bitmask,
                       tile_cnt_next, bitmask_next, cand, vals, idx, status);
        } else {
            GCE_LAUNCH(rk_emit_kernel<false>, wave_grid(lay.TT, r_emit0, r_emit0), kTkThreads, 0,
                       st, t->d_layers, t->d_tile_layer, t->tiles_pw, W, ncomp, t->N, t->vals_pw,
                       t->comp_N, grad, mem, eta, segs, nullptr, tile_cnt, bitmask, nullptr,
                       nullptr, cand, vals, idx, status);
        }
        if (check_launch() != GCE_OK) return GCE_ERR_CUDA;
        if (pipe) {
            std::lock_guard<std::mutex> lk(t->rk_mu);
            t->rk_ws = ws;
            t->rk_seed = seed;
            t->rk_step = step + 1;
            t->rk_W = W;
            t->rk_worker0 = worker0;
            t->rk_valid = true;
        }
    }
    return launch_dense_layers(t, W, grad, mem, eta, vals, status, st);
}

extern "C" int ef_randk_step(const gce_table* t, int32_t W, const float* grad, float* mem, float eta,
                             const int32_t* k_or_rank, uint64_t seed, uint64_t step, float* vals,
                             int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
    return randk_step(t, W, 0, grad, mem, eta, k_or_rank, seed, step, vals, idx, ws, ws_bytes,
                      stream);
}

extern "C" int ef_randk_step_at(const gce_table* t, int64_t worker0, int32_t W, const float* grad,
                                float* mem, float eta, const int32_t* k_or_rank, uint64_t seed,
                                uint64_t step, float* vals, int32_t* idx, void* ws,
                                size_t ws_bytes, void* stream) {
    return randk_step(t, W, worker0, grad, mem, eta, k_or_rank, seed, step, vals, idx, ws,
                      ws_bytes, stream);
}
