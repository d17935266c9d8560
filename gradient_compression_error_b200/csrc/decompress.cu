// decompress.cu -- aggregate of W workers' compressed payloads into one dense
// fp32 buffer, on sm_100a.
//
// "On the Utility of Gradient Compression in Distributed Training Systems",
// Method / Key results: the workers' compressed gradients are combined
// (all-reduce for PowerSGD, gather for sparse payloads); here the W data-
// parallel replicas live in one GPU's HBM and the combination is a sum in
// worker order from +0.0 with fp32 round-to-nearest adds, times `scale`.
//
// Design: every output element is written once, after all workers'
// contributions to it are summed on chip in worker order.  Sparse payloads
// are sorted by index, so a first pass (bounds) turns each (worker, layer)
// list into per-span entry ranges (1024 outputs a span) by comparing
// neighbouring indices -- no searching; then a warp per span gathers its
// entries and adds them into its own shared accumulator (dc_sparse_kernel).
// Sign payloads of up to 8 workers are decoded by table lookup
// (dc_sign8_kernel); other layers and more workers take a block per
// 4096-output tile (dc_accum_kernel, dc_sign_kernel).  DRAM traffic: the
// payload read once plus one 4-byte write per output element.
#include <mutex>

#include "common.cuh"
#include "scan.cuh"

namespace gce {

constexpr int kDcThreads = 128;                   // 4 warps per decode tile
static_assert(kDcSpan * (kDcThreads / 32) == kDcTile, "a warp owns one span of a tile");

size_t decompress_ws_bytes(const gce_table* t, int32_t W) {
    Carver c;
    c.take<int32_t>(int64_t(W) * t->dc_slots);
    return c.off;
}

__device__ __forceinline__ int32_t layer_k(const DevLayer& L, const int32_t* k_or_rank, int32_t l) {
    const int32_t k = k_or_rank ? k_or_rank[l] : L.cap;
    return (k >= 1 && k <= L.cap) ? k : 0;  // out of range: the layer contributes nothing
}

// bounds[w][L.dc_base + ss] = first payload entry of (w, l) whose index lies in
// decode span ss (1024 outputs) or later; slot nspans holds k.  A thread takes
// kDcBoundPer consecutive entries (two 16-byte loads when the payload slice is
// aligned) and the entry before them, and writes the slots of the spans that
// begin after an entry's predecessor and at or before the entry itself.
constexpr int kDcBoundPer = 8;

__global__ void __launch_bounds__(256, 8) dc_bounds_kernel(const DevLayer* __restrict__ layers,
                                                        const int32_t* __restrict__ bunit_layer,
                                                        const int32_t* __restrict__ bunit_chunk,
                                                        int32_t bunits_pw, int32_t W,
                                                        int64_t vals_pw, int32_t dc_slots,
                                                        const int32_t* __restrict__ k_or_rank,
                                                        const int32_t* __restrict__ idx,
                                                        int32_t* __restrict__ bounds) {
    grid_dependency_sync();
    const int64_t total = int64_t(bunits_pw) * W;
    for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
        const int w = int(u / bunits_pw);
        const int bu = int(u - int64_t(w) * bunits_pw);
        const int32_t l = bunit_layer[bu];
        const DevLayer L = layers[l];
        const int32_t k = layer_k(L, k_or_rank, l);
        int32_t* b = bounds + int64_t(w) * dc_slots + L.dc_base;
        const int32_t nt = int32_t((L.n + kDcSpan - 1) >> kDcSpanLog);  // spans of the layer
        const int64_t j0 = int64_t(bunit_chunk[bu]) * kDcBoundChunk;
        if (k == 0) {
            if (j0 == 0)
                for (int32_t tt = threadIdx.x; tt <= nt; tt += blockDim.x) b[tt] = 0;
            continue;
        }
        const int32_t* ix = idx + int64_t(w) * vals_pw + L.val_off;
        const int64_t j1 = min64(j0 + kDcBoundChunk, k);
        const bool vec = (reinterpret_cast<uintptr_t>(ix) & 15) == 0;
        for (int64_t jb = j0 + int64_t(kDcBoundPer) * threadIdx.x; jb < j1;
             jb += int64_t(kDcBoundPer) * blockDim.x) {
            int32_t cur[kDcBoundPer];
            if (vec && jb + kDcBoundPer <= j1) {
                const int4 x0 = __ldcg(reinterpret_cast<const int4*>(ix + jb));
                const int4 x1 = __ldcg(reinterpret_cast<const int4*>(ix + jb) + 1);
                cur[0] = x0.x; cur[1] = x0.y; cur[2] = x0.z; cur[3] = x0.w;
                cur[4] = x1.x; cur[5] = x1.y; cur[6] = x1.z; cur[7] = x1.w;
            } else {
#pragma unroll
                for (int q = 0; q < kDcBoundPer; ++q) cur[q] = jb + q < j1 ? __ldcg(ix + jb + q) : 0;
            }
            // span of the previous entry (-1 before the first)
            int32_t tp = jb > 0 ? min(max(__ldcg(ix + jb - 1), 0) >> kDcSpanLog, nt) : -1;
#pragma unroll
            for (int q = 0; q < kDcBoundPer; ++q) {
                if (jb + q >= j1) break;
                const int32_t j = int32_t(jb + q);
                const int32_t tj = min(max(cur[q], 0) >> kDcSpanLog, nt);
                for (int32_t tt = tp + 1; tt <= tj; ++tt) b[tt] = j;
                if (j == k - 1)
                    for (int32_t tt = tj + 1; tt <= nt; ++tt) b[tt] = k;
                tp = tj;
            }
        }
    }
}

// The entries of every worker that fall in this warp's span (outputs [start,
// start + kDcSpan) of a layer) added to the span's accumulator in worker order.
// Lane w < W holds worker w's entry range [a, a + c) of the span (from the span
// bounds); the warp walks the W ranges one after the other, 32 entries a round,
// each entry's index and value loaded into a lane.  The loads of kDcRounds
// rounds are issued before any of their adds (a round's lanes and addresses
// follow from the bounds alone), then each round adds its entries worker by
// worker (within one worker the indices are distinct, so its lanes add without
// conflict).  Run by a full warp; W <= 32.
constexpr int kDcRounds = 3;

__device__ __forceinline__ void dc_add_span(float* acc, int64_t start, int W, int32_t a,
                                            int32_t c, const float* __restrict__ vals,
                                            const int32_t* __restrict__ idx, int64_t vals_pw,
                                            int64_t val_off) {
    const int lane = threadIdx.x & 31;
    const int32_t incl = warp_inclusive_scan(c);
    const int32_t excl = incl - c;
    const int32_t total = __shfl_sync(kFull, incl, 31);
    for (int32_t q0 = 0; q0 < total; q0 += 32 * kDcRounds) {
        int w[kDcRounds];
        int32_t i[kDcRounds];
        float v[kDcRounds];
#pragma unroll
        for (int r = 0; r < kDcRounds; ++r) {
            w[r] = 0;
            i[r] = 0;
            v[r] = 0.0f;
            if (q0 + 32 * r < total) {  // the same for the whole warp
                const int32_t q = q0 + 32 * r + lane;
                int ww = 0;
#pragma unroll
                for (int step = 16; step > 0; step >>= 1) {
                    const int32_t e = __shfl_sync(kFull, excl, min(ww + step, 31));
                    if (ww + step < W && e <= q) ww += step;
                }
                const int32_t aw = __shfl_sync(kFull, a, ww), ew = __shfl_sync(kFull, excl, ww);
                w[r] = ww;
                if (q < total) {
                    const int64_t o = int64_t(ww) * vals_pw + val_off + aw + (q - ew);
                    i[r] = int32_t(int64_t(__ldcg(idx + o)) - start);
                    v[r] = __ldcg(vals + o);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kDcRounds; ++r) {
            const bool have = q0 + 32 * r + lane < total;
            unsigned pending = __ballot_sync(kFull, have);
            while (pending) {
                const int wl = __shfl_sync(kFull, w[r], __ffs(pending) - 1);
                const bool mine = have && w[r] == wl;
                if (mine) acc[i[r]] = __fadd_rn(acc[i[r]], v[r]);
                __syncwarp();
                pending &= ~__ballot_sync(kFull, mine);
            }
        }
    }
}

// Write a span's `cnt` outputs from the warp's accumulator and zero it for the
// next span: out = fl(scale * sum), or with kApply x = fl(x - fl(scale * sum)).
// Run by a full warp after __syncwarp.
template <bool kApply>
__device__ __forceinline__ void dc_write_span(float* acc, float* o, int cnt, float scale,
                                              bool aligned) {
    const int lane = threadIdx.x & 31;
    if (aligned && cnt == kDcSpan) {
        float4* a4 = reinterpret_cast<float4*>(acc);
        float4* o4 = reinterpret_cast<float4*>(o);
#pragma unroll
        for (int j = 0; j < kDcSpan / 4 / 32; ++j) {
            const float4 x = a4[lane + 32 * j];
            __stcs(o4 + lane + 32 * j, dc_final4<kApply>(x, scale, o4 + lane + 32 * j));
            a4[lane + 32 * j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    } else {
        for (int i = lane; i < kDcSpan; i += 32) {
            if (i < cnt) o[i] = dc_final<kApply>(acc[i], scale, o + i);
            acc[i] = 0.0f;
        }
    }
    __syncwarp();
}

// TOPK and RANDK tiles for W <= 32 workers.  Each warp owns one 1024-output span
// at a time (four spans to a decode tile) with its own accumulator in shared
// memory: it reads the span's entry bounds of every worker, adds the entries in
// worker order and writes the span out.  No warp waits for another; the next
// span's tile record is loaded while the current span is added, so a span's
// chain of dependent loads is its bounds and then its entries.
template <bool kApply>
__global__ void __launch_bounds__(kDcThreads, kApply ? 9 : 10) dc_sparse_kernel(
    const DcTileInfo* __restrict__ tiles, int32_t ntiles, int32_t W, int64_t vals_pw,
    int32_t dc_slots, const int32_t* __restrict__ k_or_rank, const float* __restrict__ vals,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ bounds, float scale,
    float* __restrict__ out) {
    grid_dependency_sync();
    constexpr int kParts = kDcTile >> kDcSpanLog;  // spans per tile, one per warp of a block
    __shared__ __align__(16) float acc_all[kDcTile];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* acc = acc_all + warp * kDcSpan;
    for (int i = lane; i < kDcSpan / 4; i += 32)
        reinterpret_cast<float4*>(acc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncwarp();
    const int64_t nspans = int64_t(ntiles) * kParts;
    const int64_t qstep = int64_t(gridDim.x) * kParts;
    int64_t q = int64_t(blockIdx.x) * kParts + warp;
    DcTileInfo nx{};
    if (q < nspans) nx = tiles[q / kParts];
    for (; q < nspans; q += qstep) {
        const DcTileInfo T = nx;
        if (q + qstep < nspans) nx = tiles[(q + qstep) / kParts];  // the next span's record
        const int p = int(q % kParts);
        const int cnt = min(kDcSpan, T.cnt - p * kDcSpan);
        if (cnt <= 0) continue;
        int32_t k = k_or_rank ? k_or_rank[T.layer] : T.cap;
        k = (k >= 1 && k <= T.cap) ? k : 0;  // out of range: the layer contributes nothing
        int32_t a = 0, c = 0;
        if (lane < W) {
            const int32_t* b = bounds + int64_t(lane) * dc_slots + T.bslot + p;
            a = min(max(b[0], 0), k);
            c = min(max(b[1], a), k) - a;
        }
        const int64_t span0 = int64_t(T.tstart) + p * kDcSpan;
        dc_add_span(acc, span0, W, a, c, vals, idx, vals_pw, T.val_off);
        __syncwarp();
        const int64_t o = T.out_off + p * kDcSpan;
        dc_write_span<kApply>(acc, out + o, cnt, scale, (o & 3) == 0);
    }
}

template <bool kApply>
__global__ void __launch_bounds__(kDcThreads, 9) dc_accum_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ dc_tile_layer,
    const int32_t* __restrict__ tile_list, int32_t dc_tiles, int32_t W, int64_t vals_pw,
    int64_t P_pw, int64_t Q_pw, int32_t dc_slots, const int32_t* __restrict__ k_or_rank,
    const float* __restrict__ vals, const int32_t* __restrict__ idx, const float* __restrict__ P,
    const float* __restrict__ Q, const int32_t* __restrict__ bounds, float scale,
    float* __restrict__ out) {
    grid_dependency_sync();
    __shared__ __align__(16) float acc[kDcTile];
    // the accumulator is all zero between sparse tiles
    for (int i = threadIdx.x; i < kDcTile / 4; i += blockDim.x)
        reinterpret_cast<float4*>(acc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    for (int32_t u = blockIdx.x; u < dc_tiles; u += gridDim.x) {
        const int32_t t = tile_list ? tile_list[u] : u;
        const int32_t l = dc_tile_layer[t];
        const DevLayer L = layers[l];
        const int32_t tt = t - L.dc_tile0;
        const int64_t start = int64_t(tt) << kDcTileLog;
        const int cnt = int(min64(kDcTile, L.n - start));
        float* o = out + L.offset + start;
        if (L.kind == GCE_KIND_TOPK || L.kind == GCE_KIND_RANDK) {
            const int32_t k = layer_k(L, k_or_rank, l);
            // more than 32 workers (dc_sparse_kernel takes the rest): one worker
            // at a time, straight from memory
            for (int w = 0; w < W; ++w) {
                __syncthreads();
                const int32_t* b = bounds + int64_t(w) * dc_slots + L.dc_base;
                const int32_t s0 = tt << (kDcTileLog - kDcSpanLog);
                const int32_t s1 = min(s0 + (kDcTile >> kDcSpanLog),
                                       int32_t((L.n + kDcSpan - 1) >> kDcSpanLog));
                const int32_t a = min(max(b[s0], 0), k), e = min(max(b[s1], a), k);
                const float* v = vals + int64_t(w) * vals_pw + L.val_off;
                const int32_t* ix = idx + int64_t(w) * vals_pw + L.val_off;
                for (int32_t j = a + threadIdx.x; j < e; j += blockDim.x) {
                    const int64_t i = int64_t(ix[j]) - start;
                    if (i >= 0 && i < cnt) acc[i] = __fadd_rn(acc[i], v[j]);
                }
            }
            __syncthreads();
            for (int i = threadIdx.x; i < cnt; i += blockDim.x)
                o[i] = dc_final<kApply>(acc[i], scale, o + i);
            __syncthreads();
            // leave the accumulator at zero for the next sparse tile
            for (int i = threadIdx.x; i < kDcTile / 4; i += blockDim.x)
                reinterpret_cast<float4*>(acc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            __syncthreads();
        } else if (L.kind == GCE_KIND_DENSE) {
            for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
                float s = 0.0f;
                for (int w = 0; w < W; ++w)
                    s = __fadd_rn(s, vals[int64_t(w) * vals_pw + L.val_off + start + i]);
                o[i] = dc_final<kApply>(s, scale, o + i);
            }
        } else {  // POWERSGD: P Q^T over the first r columns
            const int32_t r = layer_k(L, k_or_rank, l);
            const int cap = L.cap;
            // neighbouring threads take neighbouring columns (coalesced Q
            // reads and output writes); one 32-bit division per thread finds
            // its first (row, col), then the column advances by the block size
            const uint32_t cols = uint32_t(L.cols);
            const uint32_t c0 = uint32_t((start + threadIdx.x) % int64_t(cols));
            int64_t row = (start + threadIdx.x) / int64_t(cols);
            uint32_t col = c0;
            for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
                float s = 0.0f;
                for (int w = 0; w < W; ++w) {
                    const float* p = P + int64_t(w) * P_pw + L.p_off + row * cap;
                    const float* qq = Q + int64_t(w) * Q_pw + L.q_off + int64_t(col) * cap;
                    float m = 0.0f;
                    if (r > 0) {
                        m = __fmul_rn(p[0], qq[0]);
                        for (int j = 1; j < r; ++j) m = __fmaf_rn(p[j], qq[j], m);
                    }
                    s = __fadd_rn(s, m);
                }
                o[i] = dc_final<kApply>(s, scale, o + i);
                col += blockDim.x;
                if (col >= cols) {
                    row += col / cols;
                    col %= cols;
                }
            }
        }
    }
}

// Decode of a SIGN table (SIGN and DENSE layers), one 4096-output tile per
// block.  The tile's sign words of up to 32 workers at a time are staged in
// shared memory (128 words a worker) with their scales; each thread then forms
// its 32 outputs (four neighbouring ones in each of 8 rounds) as the
// worker-order sum of +-s.
template <bool kApply>
__global__ void __launch_bounds__(kDcThreads) dc_sign_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ dc_tile_layer,
    int32_t dc_tiles, int32_t W, int64_t vals_pw, const float* __restrict__ vals, float scale,
    float* __restrict__ out) {
    grid_dependency_sync();
    constexpr int kWordsPerTile = kDcTile / 32;           // 128
    constexpr int kRounds = kDcTile / (4 * kDcThreads);   // 8
    __shared__ uint32_t sw[32 * kWordsPerTile];
    __shared__ float s_sc[32];
    for (int32_t u = blockIdx.x; u < dc_tiles; u += gridDim.x) {
        const int32_t l = dc_tile_layer[u];
        const DevLayer L = layers[l];
        const int64_t start = int64_t(u - L.dc_tile0) << kDcTileLog;
        const int cnt = int(min64(kDcTile, L.n - start));
        float* o = out + L.offset + start;
        if (L.kind == GCE_KIND_DENSE) {
            for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
                float s = 0.0f;
                for (int w = 0; w < W; ++w)
                    s = __fadd_rn(s, vals[int64_t(w) * vals_pw + L.val_off + start + i]);
                o[i] = dc_final<kApply>(s, scale, o + i);
            }
            continue;
        }
        if (L.kind != GCE_KIND_SIGN) continue;
        const int nwords = (cnt + 31) >> 5;
        const int64_t word0 = start >> 5;
        float a[kRounds][4];
#pragma unroll
        for (int it = 0; it < kRounds; ++it)
#pragma unroll
            for (int j = 0; j < 4; ++j) a[it][j] = 0.0f;
        for (int wc = 0; wc < W; wc += 32) {
            const int wn = min(32, W - wc);
            __syncthreads();  // the previous words are consumed
            // kB loads a thread in flight, then their stores
            constexpr int kB = 8;
            for (int q0 = 0; q0 < wn * nwords; q0 += kB * kDcThreads) {
                uint32_t v[kB];
#pragma unroll
                for (int e = 0; e < kB; ++e) {
                    const int q = q0 + e * kDcThreads + int(threadIdx.x);
                    v[e] = 0u;
                    if (q < wn * nwords) {
                        const int wq = q / nwords, j = q - wq * nwords;
                        v[e] = reinterpret_cast<const uint32_t*>(
                            vals + int64_t(wc + wq) * vals_pw + L.val_off + 4)[word0 + j];
                    }
                }
#pragma unroll
                for (int e = 0; e < kB; ++e) {
                    const int q = q0 + e * kDcThreads + int(threadIdx.x);
                    if (q < wn * nwords) {
                        const int wq = q / nwords;
                        sw[wq * kWordsPerTile + (q - wq * nwords)] = v[e];
                    }
                }
            }
            if (int(threadIdx.x) < wn)
                s_sc[threadIdx.x] = vals[int64_t(wc + threadIdx.x) * vals_pw + L.val_off];
            __syncthreads();
            for (int wq = 0; wq < wn; ++wq) {
                const float sc = s_sc[wq];
#pragma unroll
                for (int it = 0; it < kRounds; ++it) {
                    const int i = 4 * int(threadIdx.x) + 4 * kDcThreads * it;
                    const uint32_t nib = sw[wq * kWordsPerTile + (i >> 5)] >> (i & 31);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        a[it][j] = __fadd_rn(a[it][j], ((nib >> j) & 1u) ? -sc : sc);
                }
            }
        }
        const bool al = ((L.offset + start) & 3) == 0;
#pragma unroll
        for (int it = 0; it < kRounds; ++it) {
            const int i = 4 * int(threadIdx.x) + 4 * kDcThreads * it;
            if (al && i + 4 <= cnt) {
                float4* o4 = reinterpret_cast<float4*>(o + i);
                __stcs(o4, dc_final4<kApply>(make_float4(a[it][0], a[it][1], a[it][2], a[it][3]),
                                             scale, o4));
            } else {
                for (int j = 0; j < 4; ++j)
                    if (i + j < cnt) o[i + j] = dc_final<kApply>(a[it][j], scale, o + i + j);
            }
        }
    }
}

// Decode of a SIGN table (SIGN and DENSE layers) for W <= 8 workers.  An
// output's W sign bits pick one of 2^W worker-order sums of +-s_w, so the
// block forms that table once per layer -- each entry by the same fp32 adds
// from +0.0 in worker order as the output's own sum, then times `scale` -- and
// an output is one lookup.  A warp takes four sign words (128 outputs) of every
// worker at a time: lane 8c + w holds worker w's word c, and after a 32 x 32
// bit transpose lane b holds bit b of all 32 words, whose byte c is the W-bit
// pattern of output 32c + b.  Each block decodes a contiguous run of tiles, so
// the table is rebuilt only where the layer changes.
template <bool kApply>
__global__ void __launch_bounds__(kDcThreads) dc_sign8_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ dc_tile_layer,
    int32_t dc_tiles, int32_t W, int64_t vals_pw, const float* __restrict__ vals, float scale,
    float* __restrict__ out) {
    grid_dependency_sync();
    constexpr int kWarps = kDcThreads / 32;
    constexpr int kGroups = kDcTile / 128 / kWarps;  // four-word groups a warp takes per tile
    __shared__ float s_tab[256];
    __shared__ float s_sc[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wk = lane & 7, col = lane >> 3;
    const int32_t u0 = int32_t(int64_t(dc_tiles) * blockIdx.x / gridDim.x);
    const int32_t u1 = int32_t(int64_t(dc_tiles) * (blockIdx.x + 1) / gridDim.x);
    int32_t tab_layer = -1;
    for (int32_t u = u0; u < u1; ++u) {
        const int32_t l = dc_tile_layer[u];
        const DevLayer L = layers[l];
        const int64_t start = int64_t(u - L.dc_tile0) << kDcTileLog;
        const int cnt = int(min64(kDcTile, L.n - start));
        float* o = out + L.offset + start;
        if (L.kind == GCE_KIND_DENSE) {
            for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
                float s = 0.0f;
                for (int w = 0; w < W; ++w)
                    s = __fadd_rn(s, vals[int64_t(w) * vals_pw + L.val_off + start + i]);
                o[i] = dc_final<kApply>(s, scale, o + i);
            }
            continue;
        }
        if (L.kind != GCE_KIND_SIGN) continue;
        if (l != tab_layer) {  // the same for the whole block
            __syncthreads();   // the last layer's table is no longer read
            if (int(threadIdx.x) < W) s_sc[threadIdx.x] = vals[int64_t(threadIdx.x) * vals_pw + L.val_off];
            __syncthreads();
            for (int p = threadIdx.x; p < (1 << W); p += blockDim.x) {
                float s = 0.0f;
                for (int w = 0; w < W; ++w) s = __fadd_rn(s, ((p >> w) & 1) ? -s_sc[w] : s_sc[w]);
                s_tab[p] = __fmul_rn(s, scale);
            }
            __syncthreads();
            tab_layer = l;
        }
        const int nwords = (cnt + 31) >> 5;
        // worker wk's sign words of this tile (a lane with wk >= W reads none)
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(
                                 vals + int64_t(wk < W ? wk : 0) * vals_pw + L.val_off + 4) +
                             (start >> 5);
        uint32_t x[kGroups];
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
            const int c = (g * kWarps + warp) * 4 + col;  // word of the tile
            x[g] = (wk < W && c < nwords) ? __ldcg(wp + c) : 0u;
        }
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
            const uint32_t pat = warp_transpose32(x[g]);
            const int i0 = (g * kWarps + warp) * 128 + lane;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int i = i0 + 32 * c;
                if (i < cnt) {
                    const float v = s_tab[(pat >> (8 * c)) & 0xFFu];
                    o[i] = kApply ? __fsub_rn(o[i], v) : v;
                }
            }
        }
    }
}

// bounds pass plus the decode kernels for every kind the table holds;
// apply: out is the parameter vector x and gets x - scale * sum
template <bool kApply>
static int launch_decode_t(const gce_table* t, int32_t W, const float* vals, const int32_t* idx,
                           const int32_t* k_or_rank, const float* P, const float* Q, float scale,
                           float* out, int32_t* bounds, cudaStream_t st) {
    const bool sparse = t->ckind == GCE_KIND_TOPK || t->ckind == GCE_KIND_RANDK;
    static const int r_bounds = resident_blocks(dc_bounds_kernel, 256);
    static const int r_accum = resident_blocks(dc_accum_kernel<kApply>, kDcThreads);
    if (t->ckind == GCE_KIND_SIGN && W <= 8) {
        static const int r_sign8 = resident_blocks(dc_sign8_kernel<kApply>, kDcThreads);
        GCE_LAUNCH_AS(kApply ? "dc_sign8_kernel<true>" : "dc_sign8_kernel<false>",
                      dc_sign8_kernel<kApply>, wave_grid(t->dc_tiles, 16, r_sign8), kDcThreads,
                      0, st, t->d_layers, t->d_dc_tile_layer, t->dc_tiles, W, t->vals_pw, vals,
                      scale, out);
        return check_launch();
    }
    if (t->ckind == GCE_KIND_SIGN) {
        static const int r_sign = resident_blocks(dc_sign_kernel<kApply>, kDcThreads);
        const int grid = wave_grid(t->dc_tiles, 16, r_sign);
        if (kApply)
            GCE_LAUNCH(dc_sign_kernel<true>, grid, kDcThreads, 0, st, t->d_layers,
                       t->d_dc_tile_layer, t->dc_tiles, W, t->vals_pw, vals, scale, out);
        else
            GCE_LAUNCH(dc_sign_kernel<false>, grid, kDcThreads, 0, st, t->d_layers,
                       t->d_dc_tile_layer, t->dc_tiles, W, t->vals_pw, vals, scale, out);
        return check_launch();
    }
    if (sparse && t->bunits_pw > 0) {
        const int64_t units = int64_t(t->bunits_pw) * W;
        GCE_LAUNCH(dc_bounds_kernel, wave_grid(units, 8, r_bounds), 256, 0, st, t->d_layers,
                   t->d_bunit_layer, t->d_bunit_chunk, t->bunits_pw, W, t->vals_pw, t->dc_slots,
                   k_or_rank, idx, bounds);
    }
    if (sparse && W <= 32) {
        // sparse tiles by the warp-per-span kernel, DENSE tiles by the general one
        static const int r_sparse = resident_blocks(dc_sparse_kernel<kApply>, kDcThreads);
        if (t->dc_sp_n > 0)
            GCE_LAUNCH_AS(kApply ? "dc_sparse_kernel<true>" : "dc_sparse_kernel<false>",
                          dc_sparse_kernel<kApply>, wave_grid(t->dc_sp_n, 16, r_sparse),
                          kDcThreads, 0, st, t->d_dc_sp_info, t->dc_sp_n, W, t->vals_pw,
                          t->dc_slots, k_or_rank, vals, idx, bounds, scale, out);
        if (t->dc_dn_n > 0)
            GCE_LAUNCH_AS(kApply ? "dc_accum_kernel<true>" : "dc_accum_kernel<false>",
                          dc_accum_kernel<kApply>, wave_grid(t->dc_dn_n, 16, r_accum),
                          kDcThreads, 0, st, t->d_layers, t->d_dc_tile_layer, t->d_dc_dn_tiles,
                          t->dc_dn_n, W, t->vals_pw, t->P_pw, t->Q_pw, t->dc_slots, k_or_rank,
                          vals, idx, P, Q, bounds, scale, out);
        return check_launch();
    }
    // PowerSGD layers by their own tiled kernel when it takes them (then the
    // element-wise kernel covers only the other layers' tiles)
    const bool lowrank = t->nps > 0 &&
                         launch_lowrank_decode(t, W, k_or_rank, P, Q, scale, out, kApply, st);
    const int32_t ntiles = lowrank ? t->dc_nl_n : t->dc_tiles;
    const int32_t* list = lowrank ? t->d_dc_nl_tiles : nullptr;
    if (ntiles > 0) {
        const int grid = wave_grid(ntiles, 16, r_accum);
        if (kApply)
            GCE_LAUNCH(dc_accum_kernel<true>, grid, kDcThreads, 0, st, t->d_layers,
                       t->d_dc_tile_layer, list, ntiles, W, t->vals_pw, t->P_pw, t->Q_pw,
                       t->dc_slots, k_or_rank, vals, idx, P, Q, bounds, scale, out);
        else
            GCE_LAUNCH(dc_accum_kernel<false>, grid, kDcThreads, 0, st, t->d_layers,
                       t->d_dc_tile_layer, list, ntiles, W, t->vals_pw, t->P_pw, t->Q_pw,
                       t->dc_slots, k_or_rank, vals, idx, P, Q, bounds, scale, out);
    }
    return check_launch();
}

static int launch_decode(const gce_table* t, int32_t W, const float* vals, const int32_t* idx,
                         const int32_t* k_or_rank, const float* P, const float* Q, float scale,
                         float* out, int32_t* bounds, cudaStream_t st) {
    return launch_decode_t<false>(t, W, vals, idx, k_or_rank, P, Q, scale, out, bounds, st);
}

}  // namespace gce

using namespace gce;

extern "C" int decompress_accumulate(const gce_table* t, int32_t W, const float* vals,
                                     const int32_t* idx, const int32_t* k_or_rank, const float* P,
                                     const float* Q, float scale, float* out, void* ws,
                                     size_t ws_bytes, void* stream) {
    if (!t || W < 1 || !out || !ws || !aligned16(out) || !aligned16(ws)) return GCE_ERR_ARG;
    const bool sparse = t->ckind == GCE_KIND_TOPK || t->ckind == GCE_KIND_RANDK;
    if ((t->vals_pw > 0 && !vals) || (sparse && !idx)) return GCE_ERR_ARG;
    if (t->ckind == GCE_KIND_POWERSGD && (!P || !Q)) return GCE_ERR_ARG;
    if (ws_bytes < decompress_ws_bytes(t, W)) return GCE_ERR_WORKSPACE;
    return launch_decode(t, W, vals, idx, k_or_rank, P, Q, scale, out,
                         at<int32_t>(ws, GCE_WS_HEADER_BYTES), static_cast<cudaStream_t>(stream));
}

extern "C" int decompress_apply(const gce_table* t, int32_t W, const float* vals,
                                const int32_t* idx, const int32_t* k_or_rank, const float* P,
                                const float* Q, float scale, float* x, void* ws, size_t ws_bytes,
                                void* stream) {
    if (!t || W < 1 || !x || !ws || !aligned16(x) || !aligned16(ws)) return GCE_ERR_ARG;
    const bool sparse = t->ckind == GCE_KIND_TOPK || t->ckind == GCE_KIND_RANDK;
    if ((t->vals_pw > 0 && !vals) || (sparse && !idx)) return GCE_ERR_ARG;
    if (t->ckind == GCE_KIND_POWERSGD && (!P || !Q)) return GCE_ERR_ARG;
    if (ws_bytes < decompress_ws_bytes(t, W)) return GCE_ERR_WORKSPACE;
    return launch_decode_t<true>(t, W, vals, idx, k_or_rank, P, Q, scale, x,
                                 at<int32_t>(ws, GCE_WS_HEADER_BYTES),
                                 static_cast<cudaStream_t>(stream));
}

extern "C" int gce_memsgd_eta(int64_t step, double mu, double a, float* eta) {
    if (!eta || !(mu > 0.0) || !(a + double(step) > 0.0) || step < 0) return GCE_ERR_ARG;
    const double e = 8.0 / (mu * (a + double(step)));
    if (!(e < 3.0e38)) return GCE_ERR_ARG;
    *eta = float(e);
    return GCE_OK;
}

// ---- decode without a caller workspace -------------------------------------------------
// Some callers cannot hand the library a workspace: code that runs inside
// another allocator (a caching allocator's out-of-memory hook, for one), code
// whose device memory is all reserved up front by its framework, and code in
// a latency-critical loop that must not pay cudaMalloc's implicit device-wide
// synchronisation.  For them, decompress_accumulate_noalloc keeps its only
// scratch -- the per-tile entry bounds -- in the fixed array below, which the
// module reserves on every GPU that loads this library until the process
// exits.  4 MiB: W x (decode spans of 1024 elements + layers) <= 1,048,576
// bound slots (the BERT-base table at W = 8 uses 856,088).
constexpr int64_t kNoAllocBoundSlots = int64_t(1) << 20;
static __device__ __align__(256) int32_t g_noalloc_bounds[kNoAllocBoundSlots];

// Device address of g_noalloc_bounds on the current device (host code cannot
// use the symbol itself as a device address).  Looked up again on every call
// made outside stream capture, so a context re-created after cudaDeviceReset
// gets its own array's address; during capture the address of the last call
// outside capture on that device is used (the first call on a device must not
// be captured).  A failed look-up clears the runtime's error state so that it
// does not surface in a later, unrelated call.
static int32_t* noalloc_bounds_on_current_device(cudaStream_t st) {
    static std::mutex mu;
    static int32_t* addr[64] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return nullptr;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (cs == cudaStreamCaptureStatusNone || !addr[dev]) {
        if (cs != cudaStreamCaptureStatusNone) return nullptr;  // never looked up outside capture
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_bounds) != cudaSuccess || !p) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = static_cast<int32_t*>(p);
    }
    return addr[dev];
}

extern "C" int decompress_accumulate_noalloc(const gce_table* t, int32_t W, const float* vals,
                                             const int32_t* idx, const int32_t* k_or_rank,
                                             const float* P, const float* Q, float scale,
                                             float* out, void* stream) {
    if (!t || W < 1 || !out || !aligned16(out)) return GCE_ERR_ARG;
    const bool sparse = t->ckind == GCE_KIND_TOPK || t->ckind == GCE_KIND_RANDK;
    if ((t->vals_pw > 0 && !vals) || (sparse && !idx)) return GCE_ERR_ARG;
    if (t->ckind == GCE_KIND_POWERSGD && (!P || !Q)) return GCE_ERR_ARG;
    if (int64_t(W) * t->dc_slots > kNoAllocBoundSlots) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* bounds = noalloc_bounds_on_current_device(st);
    if (!bounds) return GCE_ERR_CUDA;
    // every bound slot a sparse layer uses is rewritten by the bounds pass, so
    // nothing left from an earlier call needs clearing
    return launch_decode(t, W, vals, idx, k_or_rank, P, Q, scale, out, bounds, st);
}
