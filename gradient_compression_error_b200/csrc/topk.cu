// topk.cu -- Mem-SGD error-feedback top-k step on sm_100a.
//
// "Sparsified SGD with Memory", Method: g_t = comp_k(m_t + eta*grad) and
// m_{t+1} = m_t + eta*grad - g_t, comp_k = top-k (Abstract).  The chosen set
// is the k largest |v| (ties -> lower index), emitted in ascending index;
// the memory keeps v except on the chosen set, where it becomes +0.
//
// Design (one launch per phase over every (worker, layer) of the table):
//   setup    per-layer k, clear counters and histograms
//   sample   read one 128-byte run of grad/mem per 4096 elements, histogram
//            the |v| keys and, interpolating inside the crossing bins, pick
//            two bounds with a wide statistical margin: lo (the k-th largest
//            key lies above it) and hi (almost surely chosen above it);
//            layers under 65536 elements are histogrammed whole and get
//            exact bounds (the edges of the bin holding the k-th key)
//   main     the only full pass over HBM: v = fl(m + fl(eta*g)); memory <- v,
//            or +0 when key > hi; every element with key >= lo is appended, in
//            index order within its 8192-element tile, to the layer's
//            candidate list (values and indices in two arrays)
//   units    per layer: a short list (fewer than k candidates) sends the layer
//            to the exact fallback; histogram work is cut into units
//   restore  + respill  the fallback: memory zeroed above hi gets v back
//            from the candidate list, then the layer is re-listed whole
//   hist1-3  radix levels over the candidate keys find the exact k-th largest
//            key T and how many keys equal to T to take.  Level 1 spends 3072
//            of its 4096 bins on [lo, top] (top: a sampled upper bound on T with
//            the same margin as lo) and 1024 on the keys above, so that T's bin
//            is narrow (a few hundred keys); then either the count pass lists
//            the few keys in that bin and the scan fixes T from the list (the
//            usual case), or level 2 (4096 bins over that bin) fixes it; level
//            3 has work only when T fell in a coarse bin or the layer was
//            re-listed whole (every range then needs three levels)
//   count / scan / emit   per-tile counts of key > T and key == T, a prefix
//            over the tiles (first fixing T from the list, where there is one,
//            and adding the listed keys to their tiles' counts), then the
//            ordered write of (v, i); memory +0 for
//            chosen entries at or below hi, v again for entries above hi that
//            were not chosen
// Results never depend on lo or hi.  DRAM traffic: 12 B per element (read
// grad and mem, write mem) plus about 8 B per candidate (about 1.5 % of the
// elements), the payload, and a few scattered memory writes.
#include <cmath>

#include "common.cuh"
#include "scan.cuh"
#include "topk_layout.cuh"

namespace gce {

struct TkLayout {
    int64_t S = 0, TT = 0;
    size_t segs = 0, hists = 0, unit_start = 0, unit_seg = 0, redo_list = 0, tile_dir = 0,
           tile_cnt = 0,
           spill_v = 0, spill_i = 0, total = 0;
};

static TkLayout tk_layout(const gce_table* t, int32_t W) {
    TkLayout o;
    Carver c;
    o.S = (t->ckind == GCE_KIND_TOPK) ? int64_t(W) * int64_t(t->comp.size()) : 0;
    o.TT = (t->ckind == GCE_KIND_TOPK) ? int64_t(W) * t->tiles_pw : 0;
    o.segs = c.take<TkSeg>(o.S);
    o.hists = c.take<int32_t>(o.S * (kTkSBins + 3 * kTkBins));
    o.unit_start = c.take<int32_t>(o.S + 1);
    // (segment, unit within it) of every histogram unit; a segment of n
    // candidates has ceil(n / kTkHUnit) units and n is at most the layer size
    o.unit_seg = c.take<int2>(o.S ? int64_t(W) * (t->comp_N / kTkHUnit + int64_t(t->comp.size())) : 0);
    o.redo_list = c.take<int32_t>(o.TT + 1);
    o.tile_dir = c.take<int2>(o.TT);
    o.tile_cnt = c.take<int2>(o.TT);
    o.spill_v = c.take<float>(o.S ? int64_t(W) * t->comp_N : 0);
    o.spill_i = c.take<int32_t>(o.S ? int64_t(W) * t->comp_N : 0);
    o.total = c.off;
    return o;
}

size_t topk_ws_bytes(const gce_table* t, int32_t W) { return tk_layout(t, W).total; }

// hist(level, seg): level 0 = sample (kTkSBins bins), 1..3 = radix levels (kTkBins)
__device__ __forceinline__ int32_t* tk_hist(int32_t* hists, int64_t S, int level, int64_t seg) {
    if (level == 0) return hists + seg * kTkSBins;
    return hists + S * kTkSBins + (int64_t(level - 1) * S + seg) * kTkBins;
}

// ---- setup -------------------------------------------------------------------
__global__ void __launch_bounds__(256) tk_setup_kernel(const DevLayer* __restrict__ layers,
                                                       const int32_t* __restrict__ comp,
                                                       int32_t ncomp, int64_t S,
                                                       const int32_t* __restrict__ k_or_rank,
                                                       TkSeg* __restrict__ segs,
                                                       int4* __restrict__ hists4, int64_t n4,
                                                       int32_t* __restrict__ status) {
    grid_dependency_sync();
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride)
        hists4[i] = make_int4(0, 0, 0, 0);
    for (int64_t s = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; s < S; s += stride) {
        const DevLayer L = layers[comp[s % ncomp]];
        const int32_t k = k_or_rank ? k_or_rank[comp[s % ncomp]] : L.cap;
        TkSeg g{};
        if (k >= 1 && k <= L.cap && int64_t(k) <= L.n) {
            g.k = k;
        } else {
            g.k = 0;
            set_status(status, GCE_STATUS_K_RANGE);
        }
        g.lo = 0;            // until the sample pass sets them: list every
        g.hi = 0xFFFFFFFFu;  // element and zero nothing in the main pass
        g.top = 0x7FFFFFFFu;
        segs[s] = g;
    }
}

// ---- sample + bounds ----------------------------------------------------------
__host__ __device__ inline int64_t tk_samples_in(int64_t n) {
    const int64_t nch = (n + kTkSampleStride - 1) / kTkSampleStride;
    const int64_t last = n - (nch - 1) * kTkSampleStride;
    return (nch - 1) * kTkSampleChunk + (last < kTkSampleChunk ? last : kTkSampleChunk);
}

// Sample bins of 2^19 keys (16 per octave of |v|), counted from the top.
// Lower bound: the bottom edge of the bin where `target` sampled keys are
// reached.  The density of |v| falls inside a tail bin, so interpolating
// would put this bound too high; the edge keeps the margin.  Upper bound
// (interp): linear inside the bin, which errs towards fewer keys above it --
// the safe side for a bound that only saves memory writes.  -1: not reached.
// Run by one full warp.
__device__ __forceinline__ int64_t tk_sample_key(const int32_t* h, int64_t target, bool interp) {
    int64_t above = 0;
    const int b = warp_find_from_top(h, kTkSBins, target, &above);
    if (b < 0) return -1;
    const int64_t bottom = int64_t(b) << 19;
    if (!interp) return bottom;
    const double f = double(target - above) / double(h[b]);
    const int64_t key = ((int64_t(b) + 1) << 19) - int64_t(floor(f * 524288.0));
    return key < bottom ? bottom : key;
}

__global__ void __launch_bounds__(256, 6) tk_sample_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ sunit_layer,
    const int32_t* __restrict__ sunit_part, int32_t sunits_pw, int32_t W, int32_t ncomp,
    int64_t S, int64_t N, const float* __restrict__ grad, const float* __restrict__ mem,
    float eta, TkSeg* __restrict__ segs, int32_t* __restrict__ hists, double sigma) {
    grid_dependency_sync();
    constexpr int kBatch = 8;
    __shared__ int32_t h[kTkSBins];
    __shared__ int s_last;
    const int tid = threadIdx.x;
    const int64_t total = int64_t(sunits_pw) * W;
    for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
        const int w = int(u / sunits_pw);
        const int su = int(u % sunits_pw);
        const DevLayer L = layers[sunit_layer[su]];
        const int64_t seg = int64_t(w) * ncomp + L.sidx;
        const int32_t k = segs[seg].k;
        if (k == 0) continue;
        for (int b = tid; b < kTkSBins; b += blockDim.x) h[b] = 0;
        __syncthreads();
        // a layer below kTkSampleMinN elements is histogrammed whole: its
        // bounds come from exact counts
        const bool exact = L.n < kTkSampleMinN;
        const int64_t p0 = int64_t(sunit_part[su]) * kTkSamplePart;
        const int64_t pend = min64(L.n, p0 + kTkSamplePart);
        const int64_t nch = (pend - p0 + kTkSampleStride - 1) / kTkSampleStride;
        const int64_t ne = exact ? L.n : nch * kTkSampleChunk;
        const float* g = grad + int64_t(w) * N + L.offset;
        const float* m = mem + int64_t(w) * N + L.offset;
        for (int64_t e0 = 0; e0 < ne; e0 += int64_t(kBatch) * blockDim.x) {
            float vv[kBatch];
            bool ok[kBatch];
#pragma unroll
            for (int q = 0; q < kBatch; ++q) {
                const int64_t e = e0 + int64_t(q) * blockDim.x + tid;
                const int64_t pos =
                    exact ? e : p0 + (e / kTkSampleChunk) * kTkSampleStride + (e % kTkSampleChunk);
                ok[q] = e < ne && pos < L.n;
                vv[q] = ok[q] ? residual(m[pos], eta, __ldcs(g + pos)) : 0.0f;
            }
#pragma unroll
            for (int q = 0; q < kBatch; ++q)
                if (ok[q]) atomicAdd(&h[abs_key(vv[q]) >> 19], 1);
        }
        __syncthreads();
        int32_t* gh = tk_hist(hists, S, 0, seg);
        for (int b = tid; b < kTkSBins; b += blockDim.x)
            if (h[b]) atomicAdd(gh + b, h[b]);
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            const int32_t nparts = int32_t((L.n + kTkSamplePart - 1) / kTkSamplePart);
            s_last = (atomicAdd(&segs[seg].done_s, 1) == nparts - 1);
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int b = tid; b < kTkSBins; b += blockDim.x) h[b] = __ldcg(gh + b);
            __syncthreads();
            if (tid < 32 && exact) {
                // b: the bin where the count from the top reaches k.  Fewer
                // than k keys lie above it (all chosen), at least k at or
                // above its bottom edge.
                int64_t above = 0;
                const int b = warp_find_from_top(h, kTkSBins, k, &above);
                if (tid == 0 && b >= 0) {
                    segs[seg].lo = uint32_t(b) << 19;
                    segs[seg].hi = ((uint32_t(b) + 1u) << 19) - 1u;
                    segs[seg].top = ((uint32_t(b) + 1u) << 19) - 1u;
                }
            } else if (tid < 32) {
                const int64_t ns = tk_samples_in(L.n);
                const double mu = double(k) * double(ns) / double(L.n);
                const double margin = sigma * (sqrt(mu) + 1.0);
                int64_t t_lo = int64_t(ceil(mu + margin));
                if (t_lo < 1) t_lo = 1;
                // hi aims at the expected k-th key itself: a miss either way
                // costs only a few scattered memory writes in the emit
                const int64_t t_hi = int64_t(floor(mu));
                uint32_t lo = 0, hi = 0xFFFFFFFFu;
                if (t_lo <= ns) {
                    const int64_t key = tk_sample_key(h, t_lo, false);
                    if (key > 0) lo = uint32_t(key);
                }
                if (t_hi >= 1) {
                    const int64_t key = tk_sample_key(h, t_hi, true);
                    if (key >= 0) hi = uint32_t(key);
                }
                if (hi < lo) hi = lo;  // everything zeroed above hi must be a candidate
                // top: the top edge of the bin where the count from the top
                // reaches mu - margin samples, T's upper bound with lo's margin;
                // with fewer samples than that above T, the largest sample's bin
                // (T lies above every sample with probability about e^-mu, and
                // a T above top costs a third radix level, not exactness)
                int64_t t_top = int64_t(floor(mu - margin));
                if (t_top < 1) t_top = 1;
                uint32_t top = 0x7FFFFFFFu;
                {
                    int64_t above = 0;
                    const int b = warp_find_from_top(h, kTkSBins, t_top, &above);
                    if (b >= 0) top = ((uint32_t(b) + 1u) << 19) - 1u;
                }
                if (top < lo) top = lo;
                if (tid == 0) {
                    segs[seg].lo = lo;
                    segs[seg].hi = hi;
                    segs[seg].top = top;
                }
            }
            int32_t* h1 = tk_hist(hists, S, 1, seg);  // level 1 starts at zero
            for (int b = tid; b < kTkBins; b += blockDim.x) h1[b] = 0;
        }
        __syncthreads();
    }
}

// ---- main pass -------------------------------------------------------------------------
__global__ void __launch_bounds__(kTkThreads) tk_main_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t W, int32_t ncomp, int64_t N, int64_t comp_N, const float* __restrict__ grad,
    float* __restrict__ mem, float eta, TkSeg* __restrict__ segs, int2* __restrict__ tile_dir,
    float* __restrict__ spill_v, int32_t* __restrict__ spill_i, int32_t* __restrict__ status) {
    grid_dependency_sync();
    constexpr int kIters = kTkPerThread / 4;           // 8 float4 per thread
    constexpr int kWarps = kTkThreads / 32;            // 8
    __shared__ int32_t s_wt[kIters * kWarps];
    __shared__ int32_t s_total, s_base;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t total = int64_t(tiles_pw) * W;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
        const int w = int(t / tiles_pw);
        const int lt = int(t % tiles_pw);
        const DevLayer L = layers[tile_layer[lt]];
        // keep DRAM busy through this tile's compaction: the bulk-copy engine
        // pulls this block's next tile of grad and mem into L2 meanwhile
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
        }
        const int64_t seg = int64_t(w) * ncomp + L.sidx;
        const int32_t k = segs[seg].k;
        if (k == 0) continue;
        const uint32_t lo = segs[seg].lo, hi = segs[seg].hi;
        const int64_t tstart = int64_t(lt - L.tile0) * kTkTile;
        const int cnt = int(min64(kTkTile, L.n - tstart));
        const int64_t ebase = int64_t(w) * N + L.offset + tstart;
        const float* g = grad + ebase;
        float* m = mem + ebase;
        float v[kTkPerThread];
        uint32_t flags = 0;
        if (cnt == kTkTile && (ebase & 3) == 0) {
            float4 gg[kIters], mm[kIters];
#pragma unroll
            for (int j = 0; j < kIters; ++j) {
                const int e = j * (kTkThreads * 4) + tid * 4;
                gg[j] = ld_stream4(g + e);
                mm[j] = ld_stream4(m + e);
            }
#pragma unroll
            for (int j = 0; j < kIters; ++j) {
                const int e = j * (kTkThreads * 4) + tid * 4;
                float4 x, o;
                x.x = residual(mm[j].x, eta, gg[j].x);
                x.y = residual(mm[j].y, eta, gg[j].y);
                x.z = residual(mm[j].z, eta, gg[j].z);
                x.w = residual(mm[j].w, eta, gg[j].w);
                o.x = abs_key(x.x) > hi ? 0.0f : x.x;
                o.y = abs_key(x.y) > hi ? 0.0f : x.y;
                o.z = abs_key(x.z) > hi ? 0.0f : x.z;
                o.w = abs_key(x.w) > hi ? 0.0f : x.w;
                // evict-first: the memory is not read again in this step, and
                // keeping it out of L2 leaves room for the prefetched next tile
                __stcs(reinterpret_cast<float4*>(m + e), o);
                v[4 * j + 0] = x.x;
                v[4 * j + 1] = x.y;
                v[4 * j + 2] = x.z;
                v[4 * j + 3] = x.w;
            }
#pragma unroll
            for (int q = 0; q < kTkPerThread; ++q)
                flags |= uint32_t(abs_key(v[q]) >= lo) << q;
        } else {
#pragma unroll
            for (int j = 0; j < kIters; ++j) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e = j * (kTkThreads * 4) + tid * 4 + q;
                    float x = 0.0f;
                    if (e < cnt) {
                        x = residual(m[e], eta, __ldcs(g + e));
                        m[e] = abs_key(x) > hi ? 0.0f : x;
                        flags |= uint32_t(abs_key(x) >= lo) << (4 * j + q);
                    }
                    v[4 * j + q] = x;
                }
            }
        }
        bool bad = false;
#pragma unroll
        for (int q = 0; q < kTkPerThread; ++q) bad |= abs_key(v[q]) >= kNonFiniteKey;
        flag_nonfinite(bad, status);
        // ordered compaction: element order is (j, warp, lane, q)
        int incl[kIters];
#pragma unroll
        for (int j = 0; j < kIters; ++j) {
            const int c = __popc((flags >> (4 * j)) & 0xFu);
            incl[j] = warp_inclusive_scan(c);
            if (lane == 31) s_wt[j * kWarps + warp] = incl[j];
        }
        __syncthreads();
        if (warp == 0) {
            const int a = s_wt[2 * lane], b = s_wt[2 * lane + 1];
            const int x = warp_inclusive_scan(a + b);
            const int ex = x - a - b;
            s_wt[2 * lane] = ex;
            s_wt[2 * lane + 1] = ex + a;
            if (lane == 31) s_total = x;
        }
        __syncthreads();
        if (tid == 0) {
            const int tot = s_total;
            const int base = tot ? atomicAdd(&segs[seg].spill_main, tot) : 0;
            s_base = base;
            tile_dir[t] = make_int2(base, tot);
        }
        __syncthreads();
        const int64_t sbase = int64_t(w) * comp_N + L.sp_off + s_base;
        float* ov = spill_v + sbase;
        int32_t* oi = spill_i + sbase;
#pragma unroll
        for (int j = 0; j < kIters; ++j) {
            const uint32_t f = (flags >> (4 * j)) & 0xFu;
            int pos = s_wt[j * kWarps + warp] + incl[j] - __popc(f);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (f & (1u << q)) {
                    ov[pos] = v[4 * j + q];
                    oi[pos] = int32_t(tstart + j * (kTkThreads * 4) + tid * 4 + q);
                    ++pos;
                }
            }
        }
        __syncthreads();
    }
}

// ---- units: fallback decision, tile list of the fallback, histogram units ---------------
__global__ void __launch_bounds__(1024) tk_units_kernel(const DevLayer* __restrict__ layers,
                                                        const int32_t* __restrict__ comp,
                                                        int32_t ncomp, int32_t tiles_pw,
                                                        TkSeg* __restrict__ segs, int64_t S,
                                                        int32_t* __restrict__ unit_start,
                                                        int2* __restrict__ unit_seg,
                                                        int32_t* __restrict__ redo_list,
                                                        int32_t* __restrict__ status) {
    grid_dependency_sync();
    __shared__ int s_warp[33];
    __shared__ int s_carry, s_rcarry;
    if (threadIdx.x == 0) {
        s_carry = 0;
        s_rcarry = 0;
    }
    __syncthreads();
    for (int64_t b0 = 0; b0 < S; b0 += blockDim.x) {
        const int64_t s = b0 + threadIdx.x;
        int units = 0, rtiles = 0;
        int64_t t0 = 0;
        if (s < S) {
            TkSeg& g = segs[s];
            const DevLayer L = layers[comp[s % ncomp]];
            int32_t cnt = 0;
            g.redo = 0;
            if (g.k > 0) {
                if (g.spill_main < g.k) {
                    g.redo = 1;
                    cnt = int32_t(L.n);   // the fallback lists every element
                    rtiles = L.ntiles;
                    t0 = int64_t(s / ncomp) * tiles_pw + L.tile0;
                    set_status(status, GCE_STATUS_FALLBACK);
                } else {
                    cnt = g.spill_main;
                }
                units = (cnt + kTkHUnit - 1) / kTkHUnit;
            }
            g.count = cnt;
            g.prefix = 0;
            g.width = 0;
            g.need = g.k;
        }
        int tot = 0;
        const int ex = block_exclusive_scan(units, s_warp, &tot);
        if (s < S) unit_start[s] = s_carry + ex;
        for (int i = 0; i < units; ++i) unit_seg[s_carry + ex + i] = make_int2(int32_t(s), i);
        int rtot = 0;
        const int rex = block_exclusive_scan(rtiles, s_warp, &rtot);
        for (int i = 0; i < rtiles; ++i) redo_list[1 + s_rcarry + rex + i] = int32_t(t0 + i);
        __syncthreads();
        if (threadIdx.x == 0) {
            s_carry += tot;
            s_rcarry += rtot;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        unit_start[S] = s_carry;
        redo_list[0] = s_rcarry;
    }
}

// ---- exact fallback: give v back to memory zeroed above hi, then list every element ------
__global__ void __launch_bounds__(256) tk_restore_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t ncomp, int64_t N, int64_t comp_N, const TkSeg* __restrict__ segs,
    const int32_t* __restrict__ redo_list, const int2* __restrict__ tile_dir,
    const float* __restrict__ spill_v, const int32_t* __restrict__ spill_i,
    float* __restrict__ mem) {
    grid_dependency_sync();
    const int32_t n = redo_list[0];
    for (int32_t u = blockIdx.x; u < n; u += gridDim.x) {
        const int32_t t = redo_list[1 + u];
        const int w = t / tiles_pw;
        const DevLayer L = layers[tile_layer[t % tiles_pw]];
        const uint32_t hi = segs[int64_t(w) * ncomp + L.sidx].hi;
        const int2 d = tile_dir[t];
        const int64_t sb = int64_t(w) * comp_N + L.sp_off + d.x;
        float* m = mem + int64_t(w) * N + L.offset;
        for (int j = threadIdx.x; j < d.y; j += blockDim.x) {
            const float x = spill_v[sb + j];
            if (abs_key(x) > hi) m[spill_i[sb + j]] = x;
        }
    }
}

__global__ void __launch_bounds__(256) tk_respill_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t ncomp, int64_t N, int64_t comp_N, TkSeg* __restrict__ segs,
    const int32_t* __restrict__ redo_list, int2* __restrict__ tile_dir,
    const float* __restrict__ mem, float* __restrict__ spill_v, int32_t* __restrict__ spill_i) {
    grid_dependency_sync();
    __shared__ int s_base;
    const int32_t n = redo_list[0];
    for (int32_t u = blockIdx.x; u < n; u += gridDim.x) {
        const int32_t t = redo_list[1 + u];
        const int w = t / tiles_pw;
        const int lt = t % tiles_pw;
        const DevLayer L = layers[tile_layer[lt]];
        const int64_t seg = int64_t(w) * ncomp + L.sidx;
        const int64_t tstart = int64_t(lt - L.tile0) * kTkTile;
        const int cnt = int(min64(kTkTile, L.n - tstart));
        if (threadIdx.x == 0) {
            s_base = atomicAdd(&segs[seg].spill_redo, cnt);
            tile_dir[t] = make_int2(s_base, cnt);
        }
        __syncthreads();
        const float* m = mem + int64_t(w) * N + L.offset + tstart;
        const int64_t sb = int64_t(w) * comp_N + L.sp_off + s_base;
        for (int e = threadIdx.x; e < cnt; e += blockDim.x) {
            spill_v[sb + e] = __ldcg(m + e);
            spill_i[sb + e] = int32_t(tstart + e);
        }
        __syncthreads();
    }
}

// ---- radix levels over the candidate keys ------------------------------------------------
// Smallest s with (width - 1) >> s below nb (width >= 1, nb a power of two).
__device__ __forceinline__ int tk_shift_pow2(uint32_t width, int log2_nb) {
    const int bits = 32 - __clz(width - 1u);
    return bits > log2_nb ? bits - log2_nb : 0;
}

// Level 1's bins of a segment: kTkFine bins of 2^sf keys from f0 for keys below
// f1, then kTkBins - kTkFine bins of 2^sc keys from f1 up to the largest key.
// A re-listed layer (every element a candidate) has no fine part.
struct TkL1Bins {
    uint32_t f0, f1;
    int sf, sc;
    __device__ __forceinline__ TkL1Bins(const TkSeg& g) {
        f0 = g.redo ? 0u : g.lo;
        f1 = g.redo ? 0u : g.top + 1u;  // top <= 2^31 - 1
        sf = 0;
        if (f1 > f0) {
            sf = tk_shift_pow2(f1 - f0, 12);
            while (((f1 - f0 - 1u) >> sf) >= uint32_t(kTkFine)) ++sf;
        }
        sc = f1 < 0x80000000u ? tk_shift_pow2(0x80000000u - f1, 10) : 0;
    }
    // (a listed key is never below f0; the clamp keeps any key inside the bins)
    __device__ __forceinline__ uint32_t bin(uint32_t key) const {
        return key < f1 ? min((key - f0) >> sf, uint32_t(kTkFine - 1))
                        : uint32_t(kTkFine) + ((key - f1) >> sc);
    }
    // [base, base + width) of bin b
    __device__ __forceinline__ void range(int b, uint32_t* base, uint32_t* width) const {
        if (b < kTkFine) {
            *base = f0 + (uint32_t(b) << sf);
            *width = min(f1 - *base, 1u << sf);
        } else {
            *base = f1 + (uint32_t(b - kTkFine) << sc);
            *width = min(0x80000000u - *base, 1u << sc);
        }
    }
};

template <int kLevel>
__global__ void __launch_bounds__(256, 6) tk_hist_kernel(const DevLayer* __restrict__ layers,
                                                      const int32_t* __restrict__ comp,
                                                      int32_t ncomp, int64_t S, int64_t comp_N,
                                                      TkSeg* __restrict__ segs,
                                                      const int32_t* __restrict__ unit_start,
                                                      const int2* __restrict__ unit_seg,
                                                      int32_t* __restrict__ hists,
                                                      const float* __restrict__ spill_v) {
    grid_dependency_sync();
    constexpr int kPer = 16;  // candidates per thread per load batch
    __shared__ int32_t h[kTkBins];
    __shared__ int s_last;
    const int tid = threadIdx.x;
    const int32_t total = unit_start[S];
    for (int32_t u = blockIdx.x; u < total; u += gridDim.x) {
        const int2 us = unit_seg[u];
        const int64_t s = us.x;
        const TkSeg g = segs[s];
        // levels 2 and 3 bin the range [base, base + width) that holds T; a
        // range of one key is T itself
        const uint32_t base = g.prefix, width = g.width;
        // (the same for the whole block)
        if (kLevel > 1 && (width <= 1u || g.list_mode)) continue;
        const TkL1Bins l1(g);
        const int shift = kLevel > 1 ? tk_shift_pow2(width, 12) : 0;
        const int w = int(s / ncomp);
        const DevLayer L = layers[comp[s % ncomp]];
        const int64_t j0 = int64_t(us.y) * kTkHUnit;
        for (int b = tid; b < kTkBins; b += blockDim.x) h[b] = 0;
        __syncthreads();
        const float* e = spill_v + int64_t(w) * comp_N + L.sp_off;
        for (int64_t jb = j0; jb < min64(j0 + kTkHUnit, g.count); jb += int64_t(kPer) * 256) {
            uint32_t key[kPer];
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                const int64_t j = jb + int64_t(q) * 256 + tid;
                key[q] = j < g.count ? abs_key(__ldcg(e + j)) : 0xFFFFFFFFu;
            }
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                if (key[q] == 0xFFFFFFFFu) continue;
                if (kLevel == 1) {
                    atomicAdd(&h[l1.bin(key[q])], 1);
                } else if (key[q] - base < width) {
                    atomicAdd(&h[(key[q] - base) >> shift], 1);
                }
            }
        }
        __syncthreads();
        int32_t* gh = tk_hist(hists, S, kLevel, s);
        for (int b = tid; b < kTkBins; b += blockDim.x)
            if (h[b]) atomicAdd(gh + b, h[b]);
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            int32_t* done = kLevel == 1 ? &segs[s].done_1 : (kLevel == 2 ? &segs[s].done_2 : &segs[s].done_3);
            const int32_t nunits = unit_start[s + 1] - unit_start[s];
            s_last = (atomicAdd(done, 1) == nunits - 1);
        }
        __syncthreads();
        if (s_last) {
            // the last unit of the segment: find T's bin, narrow the range
            __threadfence();
            for (int b = tid; b < kTkBins; b += blockDim.x) h[b] = __ldcg(gh + b);
            __syncthreads();
            __shared__ uint32_t s_width;
            if (tid < 32) {
                int64_t above = 0;
                const int b = warp_find_from_top(h, kTkBins, g.need, &above);
                uint32_t nb = base, nw = 1u;  // no crossing (cannot happen): stop here
                if (b >= 0) {
                    if (kLevel == 1) {
                        l1.range(b, &nb, &nw);
                    } else {
                        nb = base + (uint32_t(b) << shift);
                        nw = min(width - (uint32_t(b) << shift), 1u << shift);
                    }
                }
                // a narrow bin with few keys and room for them after the
                // candidates: the count pass lists them and the scan fixes T
                const bool list = kLevel == 1 && b >= 0 && !g.redo && nw > 1u &&
                                  nw <= uint32_t(kTkBins) && h[b] <= kTkListMax &&
                                  int64_t(g.count) + h[b] <= L.n;
                if (tid == 0) {
                    segs[s].prefix = nb;
                    segs[s].width = nw;
                    segs[s].list_mode = list ? 1 : 0;
                    if (b >= 0) segs[s].need = g.need - int32_t(above);
                    s_width = list ? 1u : nw;
                }
            }
            __syncthreads();
            // the next level's histogram of this segment starts at zero
            if (kLevel < 3 && s_width > 1u) {
                int32_t* nh = tk_hist(hists, S, kLevel + 1, s);
                for (int b = tid; b < kTkBins; b += blockDim.x) nh[b] = 0;
            }
        }
        __syncthreads();
    }
}

// ---- per-tile counts, prefix over tiles, ordered emit --------------------------------------
__global__ void __launch_bounds__(256) tk_count_kernel(const TileInfo* __restrict__ tile_info,
                                                       int32_t tiles_pw, int32_t W, int32_t ncomp,
                                                       int64_t comp_N, TkSeg* __restrict__ segs,
                                                       const int2* __restrict__ tile_dir,
                                                       int2* __restrict__ tile_cnt,
                                                       float* __restrict__ spill_v,
                                                       int32_t* __restrict__ spill_i) {
    grid_dependency_sync();
    constexpr int kBatch = 8;
    const int lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    const int64_t total = int64_t(tiles_pw) * W;
    const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (TileWalk tw(int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5), wstride, tiles_pw);
         tw.t < total; tw.next(wstride)) {
        const int64_t t = tw.t;
        const int w = tw.w, lt = tw.lt;
        const TileInfo ti = tile_info[lt];
        const int2 d = tile_dir[t];
        const int64_t s = int64_t(w) * ncomp + ti.sidx;
        const int32_t k = segs[s].k;
        int gt = 0, eq = 0;
        if (k > 0) {
            const uint32_t T = segs[s].prefix;
            // list mode: T lies in [T, T + width); keys at or above its top are
            // counted as greater and the keys inside are listed for the scan
            const bool list = segs[s].list_mode != 0;
            const uint32_t width = segs[s].width;
            const int64_t seg0 = int64_t(w) * comp_N + ti.sp_off;
            const float* e = spill_v + seg0 + d.x;
            for (int j0 = 0; j0 < d.y; j0 += 32 * kBatch) {
                uint32_t key[kBatch];
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    const int j = j0 + q * 32 + lane;
                    key[q] = j < d.y ? abs_key(__ldcg(e + j)) : 0xFFFFFFFFu;
                }
                if (!list) {
#pragma unroll
                    for (int q = 0; q < kBatch; ++q) {
                        gt += key[q] != 0xFFFFFFFFu && key[q] > T;
                        eq += key[q] == T;
                    }
                    continue;
                }
                bool any_in = false;
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    const bool valid = key[q] != 0xFFFFFFFFu;
                    gt += valid && key[q] - T >= width && key[q] > T;
                    any_in |= valid && key[q] - T < width;
                }
                if (!__any_sync(kFull, any_in)) continue;  // the usual batch
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    const bool in = key[q] != 0xFFFFFFFFu && key[q] - T < width;
                    const unsigned m = __ballot_sync(kFull, in);
                    if (m == 0u) continue;
                    int pos = 0;
                    if (lane == 0) pos = atomicAdd(&segs[s].list_n, __popc(m));
                    pos = __shfl_sync(kFull, pos, 0) + __popc(m & lt_mask);
                    if (in) {
                        const int64_t o = seg0 + segs[s].count + pos;
                        reinterpret_cast<uint32_t*>(spill_v)[o] = key[q];
                        spill_i[o] = int32_t(t);
                    }
                }
            }
            gt = warp_sum(gt);
            eq = warp_sum(eq);
        }
        if (lane == 0) tile_cnt[t] = make_int2(gt, eq);
    }
}

__global__ void __launch_bounds__(512) tk_scan_kernel(const DevLayer* __restrict__ layers,
                                                       const int32_t* __restrict__ comp,
                                                       int32_t ncomp, int64_t S, int32_t tiles_pw,
                                                       int64_t comp_N, TkSeg* __restrict__ segs,
                                                       int2* __restrict__ tile_cnt,
                                                       const float* __restrict__ spill_v,
                                                       const int32_t* __restrict__ spill_i) {
    grid_dependency_sync();
    __shared__ int s_warp[33];
    __shared__ int32_t h[kTkBins];
    __shared__ uint32_t s_key[512];
    __shared__ uint32_t s_T;
    __shared__ int32_t s_need;
    for (int64_t s = blockIdx.x; s < S; s += gridDim.x) {
        if (segs[s].k == 0) continue;
        const int w = int(s / ncomp);
        const DevLayer L = layers[comp[s % ncomp]];
        int2* tc = tile_cnt + int64_t(w) * tiles_pw + L.tile0;
        if (segs[s].list_mode) {
            // fix T from the listed keys of level 1's bin [base, base + width),
            // then add each listed key to its tile's counts
            const uint32_t base = segs[s].prefix;
            const int32_t need = segs[s].need, c = segs[s].list_n;
            const int64_t o = int64_t(w) * comp_N + L.sp_off + segs[s].count;
            const uint32_t* lk = reinterpret_cast<const uint32_t*>(spill_v) + o;
            const int32_t* lt = spill_i + o;
            if (c <= int(blockDim.x)) {
                // a short list: each key counts the keys above and equal to
                // it; T is the key whose count from the top reaches need (the
                // first thread holding it writes)
                if (threadIdx.x == 0) {
                    s_T = base;
                    s_need = need;
                }
                if (int(threadIdx.x) < c) s_key[threadIdx.x] = lk[threadIdx.x];
                __syncthreads();
                if (int(threadIdx.x) < c) {
                    const uint32_t me = s_key[threadIdx.x];
                    int gt = 0, eq = 0, eq_before = 0;
                    for (int j = 0; j < c; ++j) {
                        const uint32_t x = s_key[j];
                        gt += x > me;
                        eq += x == me;
                        eq_before += x == me && j < int(threadIdx.x);
                    }
                    if (gt < need && need <= gt + eq && eq_before == 0) {
                        s_T = me;
                        s_need = need - gt;
                    }
                }
            } else {
                for (int b = threadIdx.x; b < kTkBins; b += blockDim.x) h[b] = 0;
                __syncthreads();
                for (int i = threadIdx.x; i < c; i += blockDim.x) atomicAdd(&h[lk[i] - base], 1);
                __syncthreads();
                if (threadIdx.x < 32) {
                    int64_t above = 0;
                    const int b = warp_find_from_top(h, kTkBins, need, &above);
                    if (threadIdx.x == 0) {
                        s_T = b >= 0 ? base + uint32_t(b) : base;
                        s_need = b >= 0 ? need - int32_t(above) : need;
                    }
                }
            }
            __syncthreads();
            const uint32_t T = s_T;
            if (threadIdx.x == 0) {
                segs[s].prefix = T;
                segs[s].width = 1u;
                segs[s].need = s_need;
            }
            for (int i = threadIdx.x; i < c; i += blockDim.x) {
                const uint32_t key = lk[i];
                if (key > T) atomicAdd(&tile_cnt[lt[i]].x, 1);
                else if (key == T) atomicAdd(&tile_cnt[lt[i]].y, 1);
            }
            __syncthreads();
        }
        int carry_gt = 0, carry_eq = 0;
        for (int b0 = 0; b0 < L.ntiles; b0 += blockDim.x) {
            const int i = b0 + threadIdx.x;
            // from L2, where the atomic additions above were made
            const int2 x = i < L.ntiles ? __ldcg(tc + i) : make_int2(0, 0);
            int tg = 0, te = 0;
            const int eg = block_exclusive_scan(x.x, s_warp, &tg);
            const int ee = block_exclusive_scan(x.y, s_warp, &te);
            if (i < L.ntiles) tc[i] = make_int2(carry_gt + eg, carry_eq + ee);
            carry_gt += tg;
            carry_eq += te;
        }
    }
}


__global__ void __launch_bounds__(256, 5) tk_emit_kernel(
    const TileInfo* __restrict__ tile_info, int32_t tiles_pw,
    int32_t W, int32_t ncomp, int64_t N, int64_t comp_N, int64_t vals_pw,
    const TkSeg* __restrict__ segs, const int2* __restrict__ tile_dir,
    const int2* __restrict__ tile_cnt, const float* __restrict__ spill_v,
    const int32_t* __restrict__ spill_i, float* __restrict__ mem, float* __restrict__ vals,
    int32_t* __restrict__ idx) {
    grid_dependency_sync();
    constexpr int kBatch = 8;
    const int lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    const int64_t total = int64_t(tiles_pw) * W;
    const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (TileWalk tw(int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5), wstride, tiles_pw);
         tw.t < total; tw.next(wstride)) {
        const int64_t t = tw.t;
        const int w = tw.w, lt = tw.lt;
        const TileInfo ti = tile_info[lt];
        const int2 d = tile_dir[t];
        const int2 before = tile_cnt[t];    // (key > T, key == T) in earlier tiles
        const int64_t s = int64_t(w) * ncomp + ti.sidx;
        const int32_t k = segs[s].k;
        if (k == 0) continue;
        const uint32_t T = segs[s].prefix;
        const int32_t need = segs[s].need;  // keys equal to T that are taken
        // after the fallback the memory holds v everywhere (nothing was zeroed)
        const uint32_t hi = segs[s].redo ? 0xFFFFFFFFu : segs[s].hi;
        int sel_before = before.x + min(before.y, need);
        int eq_seen = before.y;
        const int64_t sb = int64_t(w) * comp_N + ti.sp_off + d.x;
        float* vout = vals + int64_t(w) * vals_pw + ti.val_off;
        int32_t* iout = idx + int64_t(w) * vals_pw + ti.val_off;
        float* m = mem + int64_t(w) * N + ti.offset;
        for (int j0 = 0; j0 < d.y; j0 += 32 * kBatch) {
            float ev[kBatch];
            int32_t ei[kBatch];
#pragma unroll
            for (int q = 0; q < kBatch; ++q) {
                const int j = j0 + q * 32 + lane;
                ev[q] = 0.0f;
                ei[q] = -1;
                if (j < d.y) {
                    ev[q] = __ldcg(spill_v + sb + j);
                    ei[q] = __ldcg(spill_i + sb + j);
                }
            }
#pragma unroll
            for (int q = 0; q < kBatch; ++q) {
                if (j0 + q * 32 >= d.y) break;  // the warp's remaining slots are empty
                const bool valid = ei[q] >= 0;
                const uint32_t key = abs_key(ev[q]);
                const bool is_eq = valid && key == T;
                const unsigned eq_mask = __ballot_sync(kFull, is_eq);
                const int eq_rank = eq_seen + __popc(eq_mask & lt_mask);
                const bool sel = valid && (key > T || (is_eq && eq_rank < need));
                const unsigned sel_mask = __ballot_sync(kFull, sel);
                const int pos = sel_before + __popc(sel_mask & lt_mask);
                if (sel && pos < k) {
                    vout[pos] = ev[q];
                    iout[pos] = ei[q];
                    if (key <= hi) m[ei[q]] = 0.0f;
                } else if (valid && !sel && key > hi) {
                    m[ei[q]] = ev[q];  // zeroed in the main pass but not chosen
                }
                sel_before += __popc(sel_mask);
                eq_seen += __popc(eq_mask);
            }
        }
    }
}

// ---- host ------------------------------------------------------------------------------------

}  // namespace gce

using namespace gce;

extern "C" int ef_topk_step(const gce_table* t, int32_t W, const float* grad, float* mem, float eta,
                            const int32_t* k_or_rank, float* vals, int32_t* idx, void* ws,
                            size_t ws_bytes, void* stream) {
    if (!t || W < 1 || !grad || !mem || !ws) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_TOPK && t->ckind != -1) return GCE_ERR_KIND;
    if (!aligned16(grad) || !aligned16(mem) || !aligned16(ws)) return GCE_ERR_ARG;
    if ((t->vals_pw > 0) && (!vals || !aligned16(vals))) return GCE_ERR_ARG;
    if (t->ckind == GCE_KIND_TOPK && (!idx || !aligned16(idx))) return GCE_ERR_ARG;
    if (k_or_rank && (reinterpret_cast<uintptr_t>(k_or_rank) & 3)) return GCE_ERR_ARG;
    const TkLayout lay = tk_layout(t, W);
    if (ws_bytes < lay.total) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = static_cast<int32_t*>(ws);
    if (lay.S > 0) {
        const int32_t ncomp = int32_t(t->comp.size());
        TkSeg* segs = at<TkSeg>(ws, lay.segs);
        int32_t* hists = at<int32_t>(ws, lay.hists);
        int32_t* unit_start = at<int32_t>(ws, lay.unit_start);
        int2* unit_seg = at<int2>(ws, lay.unit_seg);
        int32_t* redo_list = at<int32_t>(ws, lay.redo_list);
        int2* tile_dir = at<int2>(ws, lay.tile_dir);
        int2* tile_cnt = at<int2>(ws, lay.tile_cnt);
        float* spill_v = at<float>(ws, lay.spill_v);
        int32_t* spill_i = at<int32_t>(ws, lay.spill_i);
        // the sample histograms; the sample's last block of a segment clears
        // its level-1 histogram, and a level's last block the next level's
        // when that level has work
        const int64_t n4 = lay.S * kTkSBins / 4;

        static const int r_setup = resident_blocks(tk_setup_kernel, 256);
        static const int r_sample = resident_blocks(tk_sample_kernel, 256);
        static const int r_main = resident_blocks(tk_main_kernel, kTkThreads);
        static const int r_restore = resident_blocks(tk_restore_kernel, 256);
        static const int r_respill = resident_blocks(tk_respill_kernel, 256);
        static const int r_h1 = resident_blocks(tk_hist_kernel<1>, 256);
        static const int r_h2 = resident_blocks(tk_hist_kernel<2>, 256);
        static const int r_h3 = resident_blocks(tk_hist_kernel<3>, 256);
        static const int r_count = resident_blocks(tk_count_kernel, 256);
        static const int r_scan = resident_blocks(tk_scan_kernel, 512);
        static const int r_emit = resident_blocks(tk_emit_kernel, 256);
        GCE_LAUNCH(tk_setup_kernel, wave_grid((n4 + lay.S + 255) / 256, 8, r_setup), 256, 0, st, t->d_layers,
                   t->d_comp, ncomp, lay.S, k_or_rank, segs, reinterpret_cast<int4*>(hists), n4,
                   status);
        if (t->sunits_pw > 0)
            GCE_LAUNCH(tk_sample_kernel, wave_grid(int64_t(t->sunits_pw) * W, 8, r_sample), 256, 0, st,
                       t->d_layers, t->d_sunit_layer, t->d_sunit_part, t->sunits_pw, W, ncomp,
                       lay.S, t->N, grad, mem, eta, segs, hists,
                       option_of(t, GCE_OPT_BRACKET_SIGMA));
        GCE_LAUNCH(tk_main_kernel, wave_grid(lay.TT, r_main, r_main), kTkThreads, 0, st, t->d_layers,
                   t->d_tile_layer, t->tiles_pw, W, ncomp, t->N, t->comp_N, grad, mem, eta, segs,
                   tile_dir, spill_v, spill_i, status);
        GCE_LAUNCH(tk_units_kernel, 1, 1024, 0, st, t->d_layers, t->d_comp, ncomp, t->tiles_pw,
                   segs, lay.S, unit_start, unit_seg, redo_list, status);
        GCE_LAUNCH(tk_restore_kernel, wave_grid(lay.TT, 4, r_restore), 256, 0, st, t->d_layers, t->d_tile_layer,
                   t->tiles_pw, ncomp, t->N, t->comp_N, segs, redo_list, tile_dir, spill_v,
                   spill_i, mem);
        GCE_LAUNCH(tk_respill_kernel, wave_grid(lay.TT, 4, r_respill), 256, 0, st, t->d_layers, t->d_tile_layer,
                   t->tiles_pw, ncomp, t->N, t->comp_N, segs, redo_list, tile_dir, mem, spill_v,
                   spill_i);
        const int64_t hwork = lay.TT + lay.S;
        GCE_LAUNCH(tk_hist_kernel<1>, wave_grid(hwork, 8, r_h1), 256, 0, st, t->d_layers, t->d_comp, ncomp, lay.S,
                   t->comp_N, segs, unit_start, unit_seg, hists, spill_v);
        GCE_LAUNCH(tk_hist_kernel<2>, wave_grid(hwork, 8, r_h2), 256, 0, st, t->d_layers, t->d_comp, ncomp, lay.S,
                   t->comp_N, segs, unit_start, unit_seg, hists, spill_v);
        GCE_LAUNCH(tk_hist_kernel<3>, wave_grid(hwork, 8, r_h3), 256, 0, st, t->d_layers, t->d_comp, ncomp, lay.S,
                   t->comp_N, segs, unit_start, unit_seg, hists, spill_v);
        const int64_t wwork = (lay.TT + 7) / 8;  // a warp per tile
        GCE_LAUNCH(tk_count_kernel, wave_grid(wwork, 8, r_count), 256, 0, st, t->d_tile_info,
                   t->tiles_pw, W, ncomp, t->comp_N, segs, tile_dir, tile_cnt, spill_v, spill_i);
        GCE_LAUNCH(tk_scan_kernel, wave_grid(lay.S, 4, r_scan), 512, 0, st, t->d_layers, t->d_comp, ncomp,
                   lay.S, t->tiles_pw, t->comp_N, segs, tile_cnt, spill_v, spill_i);
        GCE_LAUNCH(tk_emit_kernel, wave_grid(wwork, 8, r_emit), 256, 0, st, t->d_tile_info,
                   t->tiles_pw, W, ncomp, t->N, t->comp_N, t->vals_pw, segs, tile_dir, tile_cnt,
                   spill_v, spill_i, mem, vals, idx);
        if (check_launch() != GCE_OK) return GCE_ERR_CUDA;
    }
    return launch_dense_layers(t, W, grad, mem, eta, vals, status, st);
}
