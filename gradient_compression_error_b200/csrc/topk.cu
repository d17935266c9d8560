// topk.cu -- Mem-SGD error-feedback top-k step on sm_100a.
//
// "Sparsified SGD with Memory", Method: g_t = comp_k(m_t + eta*grad) and
// m_{t+1} = m_t + eta*grad - g_t, comp_k = top-k (Abstract).  The chosen set
// is the k largest |v| (ties -> lower index), emitted in ascending index;
// the memory keeps v except on the chosen set, where it becomes +0.
//
// Design (one launch per phase over every (worker, layer) of the table):
//   setup   per-layer k, clear counters and histograms
//   sample  read one 128-byte run of grad/mem per 2048 elements, histogram the
//           |v| keys, and pick a lower bound lo that keeps the k-th largest
//           key above it with a wide statistical margin
//   main    the only full pass over HBM: v = fl(m + fl(eta*g)), mem <- v, and
//           every element with key >= lo is appended (in index order within
//           its 8192-element tile) to the layer's candidate list
//   respill exact fallback: a layer whose candidate list came out shorter
//           than k is re-listed whole from mem (rare; correctness never
//           depends on the sample)
//   hist1-3 three 11/11/9-bit radix levels over the candidate lists find the
//           exact k-th largest key T and how many keys equal to T to take
//   count / scan / emit   per-tile counts of key > T and key == T, a prefix
//           over the tiles, and the ordered write of (v, i) plus mem[i] = +0
// DRAM traffic is 12 B per element (read grad and mem, write mem) plus
// about 8 B per candidate (a few % of the elements) and the payload.
#include <cmath>

#include "common.cuh"
#include "scan.cuh"
#include "topk_layout.cuh"

namespace gce {

static double g_bracket_sigma = 6.0;

struct TkLayout {
    int64_t S = 0, TT = 0;
    size_t segs = 0, hists = 0, unit_start = 0, tile_dir = 0, tile_cnt = 0, spill = 0, total = 0;
};

static TkLayout tk_layout(const gce_table* t, int32_t W) {
    TkLayout o;
    Carver c;
    o.S = (t->ckind == GCE_KIND_TOPK) ? int64_t(W) * int64_t(t->comp.size()) : 0;
    o.TT = (t->ckind == GCE_KIND_TOPK) ? int64_t(W) * t->tiles_pw : 0;
    o.segs = c.take<TkSeg>(o.S);
    o.hists = c.take<int32_t>(o.S * 4 * kTkBins);
    o.unit_start = c.take<int32_t>(o.S + 1);
    o.tile_dir = c.take<int2>(o.TT);
    o.tile_cnt = c.take<int2>(o.TT);
    o.spill = c.take<TkEntry>(o.S ? int64_t(W) * t->comp_N : 0);
    o.total = c.off;
    return o;
}

size_t topk_ws_bytes(const gce_table* t, int32_t W) { return tk_layout(t, W).total; }

// hist(level, seg): level 0 = sample, 1..3 = radix levels
__device__ __forceinline__ int32_t* tk_hist(int32_t* hists, int64_t S, int level, int64_t seg) {
    return hists + (int64_t(level) * S + seg) * kTkBins;
}

// ---- setup -------------------------------------------------------------------
__global__ void __launch_bounds__(256) tk_setup_kernel(const DevLayer* __restrict__ layers,
                                                       const int32_t* __restrict__ comp,
                                                       int32_t ncomp, int64_t S,
                                                       const int32_t* __restrict__ k_or_rank,
                                                       TkSeg* __restrict__ segs,
                                                       int4* __restrict__ hists4, int64_t n4,
                                                       int32_t* __restrict__ status) {
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride)
        hists4[i] = make_int4(0, 0, 0, 0);
    for (int64_t s = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; s < S; s += stride) {
        const DevLayer L = layers[comp[s % ncomp]];
        const int32_t cap = L.cap;
        const int32_t k = k_or_rank ? k_or_rank[comp[s % ncomp]] : cap;
        TkSeg g{};
        if (k >= 1 && k <= cap && int64_t(k) <= L.n) {
            g.k = k;
        } else {
            g.k = 0;
            set_status(status, GCE_STATUS_K_RANGE);
        }
        g.lo = 0;  // layers too small to sample keep every element as a candidate
        segs[s] = g;
    }
}

// ---- sample + bracket ----------------------------------------------------------
__host__ __device__ inline int64_t tk_samples_in(int64_t n) {
    const int64_t nch = (n + kTkSampleStride - 1) / kTkSampleStride;
    const int64_t last = n - (nch - 1) * kTkSampleStride;
    return (nch - 1) * kTkSampleChunk + (last < kTkSampleChunk ? last : kTkSampleChunk);
}

__global__ void __launch_bounds__(256) tk_sample_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ sunit_layer,
    const int32_t* __restrict__ sunit_part, int32_t sunits_pw, int32_t W, int32_t ncomp,
    int64_t S, int64_t N, const float* __restrict__ grad, const float* __restrict__ mem,
    float eta, TkSeg* __restrict__ segs, int32_t* __restrict__ hists, double sigma) {
    __shared__ int32_t h[kTkBins];
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
        for (int b = tid; b < kTkBins; b += blockDim.x) h[b] = 0;
        __syncthreads();
        const int64_t p0 = int64_t(sunit_part[su]) * kTkSamplePart;
        const int64_t pend = min(L.n, p0 + kTkSamplePart);
        const int64_t nch = (pend - p0 + kTkSampleStride - 1) / kTkSampleStride;
        const int64_t ne = nch * kTkSampleChunk;
        const float* g = grad + int64_t(w) * N + L.offset;
        const float* m = mem + int64_t(w) * N + L.offset;
#pragma unroll 4
        for (int64_t e = tid; e < ne; e += blockDim.x) {
            const int64_t pos = p0 + (e / kTkSampleChunk) * kTkSampleStride + (e % kTkSampleChunk);
            if (pos < L.n) {
                const float v = residual(m[pos], eta, __ldcs(g + pos));
                atomicAdd(&h[abs_key(v) >> 20], 1);
            }
        }
        __syncthreads();
        int32_t* gh = tk_hist(hists, S, 0, seg);
        for (int b = tid; b < kTkBins; b += blockDim.x)
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
            for (int b = tid; b < kTkBins; b += blockDim.x) h[b] = __ldcg(gh + b);
            __syncthreads();
            if (tid < 32) {
                const int64_t ns = tk_samples_in(L.n);
                const double mu = double(k) * double(ns) / double(L.n);
                const double tgt = mu + sigma * (sqrt(mu) + 1.0);
                int64_t target = int64_t(ceil(tgt));
                if (target < 1) target = 1;
                uint32_t lo = 0;
                if (target <= ns) {
                    int64_t above = 0;
                    const int b = warp_find_from_top(h, kTkBins, target, &above);
                    if (b > 0) lo = uint32_t(b) << 20;
                }
                if (tid == 0) segs[seg].lo = lo;
            }
        }
        __syncthreads();
    }
}

// ---- main pass / fallback re-listing ------------------------------------------------
// kCompute: v = fl(m + fl(eta*g)) and mem <- v; otherwise v = mem (the fallback
// re-lists a whole layer whose candidate list came out shorter than k).
template <bool kCompute>
__global__ void __launch_bounds__(kTkThreads) tk_main_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t W, int32_t ncomp, int64_t N, int64_t comp_N, const float* __restrict__ grad,
    float* __restrict__ mem, float eta, TkSeg* __restrict__ segs, int2* __restrict__ tile_dir,
    TkEntry* __restrict__ spill) {
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
        const int64_t seg = int64_t(w) * ncomp + L.sidx;
        const int32_t k = segs[seg].k;
        if (k == 0) continue;
        uint32_t lo = 0;
        int32_t* counter;
        if (kCompute) {
            lo = segs[seg].lo;
            counter = &segs[seg].spill_main;
        } else {
            if (segs[seg].spill_main >= k) continue;
            counter = &segs[seg].spill_redo;
        }
        const int64_t tstart = int64_t(lt - L.tile0) * kTkTile;
        const int cnt = int(min64(kTkTile, L.n - tstart));
        const int64_t ebase = int64_t(w) * N + L.offset + tstart;
        const float* g = grad + ebase;
        float* m = mem + ebase;
        float v[kTkPerThread];
        uint32_t flags = 0;
        if (cnt == kTkTile && (ebase & 3) == 0) {
#pragma unroll
            for (int j = 0; j < kIters; ++j) {
                const int e = j * (kTkThreads * 4) + tid * 4;
                float4 x;
                if (kCompute) {
                    const float4 gg = ld_stream4(g + e);
                    const float4 mm = ld_stream4(m + e);
                    x.x = residual(mm.x, eta, gg.x);
                    x.y = residual(mm.y, eta, gg.y);
                    x.z = residual(mm.z, eta, gg.z);
                    x.w = residual(mm.w, eta, gg.w);
                    *reinterpret_cast<float4*>(m + e) = x;
                } else {
                    x = __ldcg(reinterpret_cast<const float4*>(m + e));
                }
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
                        if (kCompute) {
                            x = residual(m[e], eta, __ldcs(g + e));
                            m[e] = x;
                        } else {
                            x = __ldcg(m + e);
                        }
                        flags |= uint32_t(abs_key(x) >= lo) << (4 * j + q);
                    }
                    v[4 * j + q] = x;
                }
            }
        }
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
            const int base = tot ? atomicAdd(counter, tot) : 0;
            s_base = base;
            tile_dir[t] = make_int2(base, tot);
        }
        __syncthreads();
        TkEntry* out = spill + int64_t(w) * comp_N + L.sp_off + s_base;
#pragma unroll
        for (int j = 0; j < kIters; ++j) {
            const uint32_t f = (flags >> (4 * j)) & 0xFu;
            int pos = s_wt[j * kWarps + warp] + incl[j] - __popc(f);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (f & (1u << q)) {
                    TkEntry en;
                    en.v = v[4 * j + q];
                    en.i = int32_t(tstart + j * (kTkThreads * 4) + tid * 4 + q);
                    out[pos++] = en;
                }
            }
        }
        __syncthreads();
    }
}

// ---- histogram units ------------------------------------------------------------------
__global__ void __launch_bounds__(1024) tk_units_kernel(TkSeg* __restrict__ segs, int64_t S,
                                                        int32_t* __restrict__ unit_start,
                                                        int32_t* __restrict__ status) {
    __shared__ int s_warp[33];
    __shared__ int s_carry;
    if (threadIdx.x == 0) s_carry = 0;
    __syncthreads();
    for (int64_t b0 = 0; b0 < S; b0 += blockDim.x) {
        const int64_t s = b0 + threadIdx.x;
        int units = 0;
        if (s < S) {
            TkSeg& g = segs[s];
            int32_t cnt = 0;
            if (g.k > 0) {
                const bool redo = g.spill_main < g.k;
                cnt = redo ? g.spill_redo : g.spill_main;
                if (redo) set_status(status, GCE_STATUS_FALLBACK);
                units = (cnt + kTkHUnit - 1) / kTkHUnit;
            }
            g.count = cnt;
            g.prefix = 0;
            g.need = g.k;
        }
        int tot = 0;
        const int ex = block_exclusive_scan(units, s_warp, &tot);
        if (s < S) unit_start[s] = s_carry + ex;
        __syncthreads();
        if (threadIdx.x == 0) s_carry += tot;
        __syncthreads();
    }
    if (threadIdx.x == 0) unit_start[S] = s_carry;
}

// ---- radix levels over the candidate lists --------------------------------------------------
template <int kLevel>
__global__ void __launch_bounds__(256) tk_hist_kernel(const DevLayer* __restrict__ layers,
                                                      const int32_t* __restrict__ comp,
                                                      int32_t ncomp, int64_t S, int64_t comp_N,
                                                      TkSeg* __restrict__ segs,
                                                      const int32_t* __restrict__ unit_start,
                                                      int32_t* __restrict__ hists,
                                                      const TkEntry* __restrict__ spill) {
    constexpr int kNb = kLevel == 3 ? 512 : kTkBins;
    constexpr int kShift = kLevel == 1 ? 20 : (kLevel == 2 ? 9 : 0);
    __shared__ int32_t h[kTkBins];
    __shared__ int s_last;
    const int tid = threadIdx.x;
    const int32_t total = unit_start[S];
    for (int32_t u = blockIdx.x; u < total; u += gridDim.x) {
        int64_t lo_ = 0, hi_ = S;
        while (hi_ - lo_ > 1) {
            const int64_t mid = (lo_ + hi_) >> 1;
            if (unit_start[mid] <= u) lo_ = mid; else hi_ = mid;
        }
        const int64_t s = lo_;
        const int w = int(s / ncomp);
        const DevLayer L = layers[comp[s % ncomp]];
        const uint32_t prefix = segs[s].prefix;
        const int32_t count = segs[s].count;
        const int64_t j0 = int64_t(u - unit_start[s]) * kTkHUnit;
        const int64_t j1 = min64(j0 + kTkHUnit, count);
        for (int b = tid; b < kNb; b += blockDim.x) h[b] = 0;
        __syncthreads();
        const TkEntry* e = spill + int64_t(w) * comp_N + L.sp_off;
        for (int64_t j = j0 + tid; j < j1; j += blockDim.x) {
            const uint32_t key = abs_key(e[j].v);
            bool take = true;
            if (kLevel == 2) take = (key >> 20) == (prefix >> 20);
            if (kLevel == 3) take = (key >> 9) == (prefix >> 9);
            if (take) atomicAdd(&h[(key >> kShift) & (kNb - 1)], 1);
        }
        __syncthreads();
        int32_t* gh = tk_hist(hists, S, kLevel, s);
        for (int b = tid; b < kNb; b += blockDim.x)
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
            __threadfence();
            for (int b = tid; b < kNb; b += blockDim.x) h[b] = __ldcg(gh + b);
            __syncthreads();
            if (tid < 32) {
                int64_t above = 0;
                const int32_t need = segs[s].need;
                const int b = warp_find_from_top(h, kNb, need, &above);
                if (tid == 0 && b >= 0) {
                    segs[s].prefix = prefix | (uint32_t(b) << kShift);
                    segs[s].need = need - int32_t(above);
                }
            }
        }
        __syncthreads();
    }
}

// ---- per-tile counts, prefix over tiles, ordered emit ------------------------------------------
__global__ void __launch_bounds__(256) tk_count_kernel(const DevLayer* __restrict__ layers,
                                                       const int32_t* __restrict__ tile_layer,
                                                       int32_t tiles_pw, int32_t W, int32_t ncomp,
                                                       int64_t comp_N, const TkSeg* __restrict__ segs,
                                                       const int2* __restrict__ tile_dir,
                                                       int2* __restrict__ tile_cnt,
                                                       const TkEntry* __restrict__ spill) {
    const int lane = threadIdx.x & 31;
    const int64_t total = int64_t(tiles_pw) * W;
    const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < total; t += wstride) {
        const int w = int(t / tiles_pw);
        const int lt = int(t % tiles_pw);
        const DevLayer L = layers[tile_layer[lt]];
        const int64_t s = int64_t(w) * ncomp + L.sidx;
        const int32_t k = segs[s].k;
        int gt = 0, eq = 0;
        if (k > 0) {
            const uint32_t T = segs[s].prefix;
            const int2 d = tile_dir[t];
            const TkEntry* e = spill + int64_t(w) * comp_N + L.sp_off + d.x;
            for (int j = lane; j < d.y; j += 32) {
                const uint32_t key = abs_key(e[j].v);
                gt += key > T;
                eq += key == T;
            }
            gt = warp_sum(gt);
            eq = warp_sum(eq);
        }
        if (lane == 0) tile_cnt[t] = make_int2(gt, eq);
    }
}

__global__ void __launch_bounds__(1024) tk_scan_kernel(const DevLayer* __restrict__ layers,
                                                       const int32_t* __restrict__ comp,
                                                       int32_t ncomp, int64_t S, int32_t tiles_pw,
                                                       const TkSeg* __restrict__ segs,
                                                       int2* __restrict__ tile_cnt) {
    __shared__ int s_warp[33];
    for (int64_t s = blockIdx.x; s < S; s += gridDim.x) {
        if (segs[s].k == 0) continue;
        const int w = int(s / ncomp);
        const DevLayer L = layers[comp[s % ncomp]];
        int2* tc = tile_cnt + int64_t(w) * tiles_pw + L.tile0;
        int carry_gt = 0, carry_eq = 0;
        for (int b0 = 0; b0 < L.ntiles; b0 += blockDim.x) {
            const int i = b0 + threadIdx.x;
            const int2 x = i < L.ntiles ? tc[i] : make_int2(0, 0);
            int tg = 0, te = 0;
            const int eg = block_exclusive_scan(x.x, s_warp, &tg);
            const int ee = block_exclusive_scan(x.y, s_warp, &te);
            if (i < L.ntiles) tc[i] = make_int2(carry_gt + eg, carry_eq + ee);
            carry_gt += tg;
            carry_eq += te;
        }
    }
}

__global__ void __launch_bounds__(256) tk_emit_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t W, int32_t ncomp, int64_t N, int64_t comp_N, int64_t vals_pw,
    const TkSeg* __restrict__ segs, const int2* __restrict__ tile_dir,
    const int2* __restrict__ tile_cnt, const TkEntry* __restrict__ spill, float* __restrict__ mem,
    float* __restrict__ vals, int32_t* __restrict__ idx) {
    const int lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    const int64_t total = int64_t(tiles_pw) * W;
    const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t t = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < total; t += wstride) {
        const int w = int(t / tiles_pw);
        const int lt = int(t % tiles_pw);
        const DevLayer L = layers[tile_layer[lt]];
        const int64_t s = int64_t(w) * ncomp + L.sidx;
        const int32_t k = segs[s].k;
        if (k == 0) continue;
        const uint32_t T = segs[s].prefix;
        const int32_t need = segs[s].need;  // keys equal to T that are taken
        const int2 d = tile_dir[t];
        const int2 before = tile_cnt[t];    // (key > T, key == T) in earlier tiles
        int sel_before = before.x + min(before.y, need);
        int eq_seen = before.y;
        const TkEntry* e = spill + int64_t(w) * comp_N + L.sp_off + d.x;
        float* vout = vals + int64_t(w) * vals_pw + L.val_off;
        int32_t* iout = idx + int64_t(w) * vals_pw + L.val_off;
        float* m = mem + int64_t(w) * N + L.offset;
        for (int j0 = 0; j0 < d.y; j0 += 32) {
            const int j = j0 + lane;
            TkEntry en{0.0f, 0};
            uint32_t key = 0;
            const bool valid = j < d.y;
            if (valid) {
                en = e[j];
                key = abs_key(en.v);
            }
            const bool is_eq = valid && key == T;
            const unsigned eq_mask = __ballot_sync(kFull, is_eq);
            const int eq_rank = eq_seen + __popc(eq_mask & lt_mask);
            const bool sel = valid && (key > T || (is_eq && eq_rank < need));
            const unsigned sel_mask = __ballot_sync(kFull, sel);
            const int pos = sel_before + __popc(sel_mask & lt_mask);
            if (sel && pos < k) {
                vout[pos] = en.v;
                iout[pos] = en.i;
                m[en.i] = 0.0f;
            }
            sel_before += __popc(sel_mask);
            eq_seen += __popc(eq_mask);
        }
    }
}

// ---- host ------------------------------------------------------------------------------------
template <class K>
static int occupancy(K kernel, int threads) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1)
        n = 1;
    return n;
}

static int grid_for(int64_t work, int per_sm) {
    const int64_t cap = int64_t(sm_count()) * per_sm;
    return int(max64(1, min64(work, cap)));
}

}  // namespace gce

using namespace gce;

extern "C" int gce_set_bracket_sigma(double sigma) {
    if (!(sigma > -100.0 && sigma < 100.0)) return GCE_ERR_ARG;
    g_bracket_sigma = sigma;
    return GCE_OK;
}

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
        int2* tile_dir = at<int2>(ws, lay.tile_dir);
        int2* tile_cnt = at<int2>(ws, lay.tile_cnt);
        TkEntry* spill = at<TkEntry>(ws, lay.spill);
        const int64_t n4 = lay.S * 4 * kTkBins / 4;

        GCE_LAUNCH(tk_setup_kernel, grid_for((n4 + lay.S + 255) / 256, 8), 256, 0, st, t->d_layers,
                   t->d_comp, ncomp, lay.S, k_or_rank, segs, reinterpret_cast<int4*>(hists), n4,
                   status);
        if (t->sunits_pw > 0)
            GCE_LAUNCH(tk_sample_kernel, grid_for(int64_t(t->sunits_pw) * W, 8), 256, 0, st,
                       t->d_layers, t->d_sunit_layer, t->d_sunit_part, t->sunits_pw, W, ncomp,
                       lay.S, t->N, grad, mem, eta, segs, hists, g_bracket_sigma);
        static int occ_main = occupancy(tk_main_kernel<true>, kTkThreads);
        static int occ_redo = occupancy(tk_main_kernel<false>, kTkThreads);
        GCE_LAUNCH(tk_main_kernel<true>, grid_for(lay.TT, occ_main), kTkThreads, 0, st, t->d_layers,
                   t->d_tile_layer, t->tiles_pw, W, ncomp, t->N, t->comp_N, grad, mem, eta, segs,
                   tile_dir, spill);
        GCE_LAUNCH(tk_main_kernel<false>, grid_for(lay.TT, occ_redo), kTkThreads, 0, st,
                   t->d_layers, t->d_tile_layer, t->tiles_pw, W, ncomp, t->N, t->comp_N, grad, mem,
                   eta, segs, tile_dir, spill);
        GCE_LAUNCH(tk_units_kernel, 1, 1024, 0, st, segs, lay.S, unit_start, status);
        const int hgrid = grid_for(lay.TT + lay.S, 8);
        GCE_LAUNCH(tk_hist_kernel<1>, hgrid, 256, 0, st, t->d_layers, t->d_comp, ncomp, lay.S,
                   t->comp_N, segs, unit_start, hists, spill);
        GCE_LAUNCH(tk_hist_kernel<2>, hgrid, 256, 0, st, t->d_layers, t->d_comp, ncomp, lay.S,
                   t->comp_N, segs, unit_start, hists, spill);
        GCE_LAUNCH(tk_hist_kernel<3>, hgrid, 256, 0, st, t->d_layers, t->d_comp, ncomp, lay.S,
                   t->comp_N, segs, unit_start, hists, spill);
        const int wgrid = grid_for((lay.TT + 7) / 8, 8);
        GCE_LAUNCH(tk_count_kernel, wgrid, 256, 0, st, t->d_layers, t->d_tile_layer, t->tiles_pw,
                   W, ncomp, t->comp_N, segs, tile_dir, tile_cnt, spill);
        GCE_LAUNCH(tk_scan_kernel, grid_for(lay.S, 2), 1024, 0, st, t->d_layers, t->d_comp, ncomp,
                   lay.S, t->tiles_pw, segs, tile_cnt);
        GCE_LAUNCH(tk_emit_kernel, wgrid, 256, 0, st, t->d_layers, t->d_tile_layer, t->tiles_pw, W,
                   ncomp, t->N, t->comp_N, t->vals_pw, segs, tile_dir, tile_cnt, spill, mem, vals,
                   idx);
        if (check_launch() != GCE_OK) return GCE_ERR_CUDA;
    }
    return launch_dense_layers(t, W, grad, mem, eta, vals, st);
}

namespace gce {
double bracket_sigma() { return g_bracket_sigma; }
}  // namespace gce
