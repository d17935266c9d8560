// decompress.cu -- aggregate of W workers' compressed payloads into one dense
// fp32 buffer, on sm_100a.
//
// "On the Utility of Gradient Compression in Distributed Training Systems",
// Method / Key results: the workers' compressed gradients are combined
// (all-reduce for PowerSGD, gather for sparse payloads); here the W data-
// parallel replicas live in one GPU's HBM and the combination is a sum in
// worker order from +0.0 with fp32 round-to-nearest adds, times `scale`.
//
// Design: each CTA owns one 4096-element tile of the output and accumulates
// every worker's contribution to it in shared memory, in worker order, then
// writes the tile once.  Sparse payloads are sorted by index, so a first
// pass (bounds) turns each (worker, layer) list into per-tile entry ranges
// by comparing neighbouring indices -- no searching.  DRAM traffic: the
// payload read once plus one 4-byte write per output element.
#include <mutex>

#include "common.cuh"
#include "scan.cuh"

namespace gce {

constexpr int kDcStage = 2048;  // payload entries staged in shared memory per tile

size_t decompress_ws_bytes(const gce_table* t, int32_t W) {
    Carver c;
    c.take<int32_t>(int64_t(W) * t->dc_slots);
    return c.off;
}

__device__ __forceinline__ int32_t layer_k(const DevLayer& L, const int32_t* k_or_rank, int32_t l) {
    const int32_t k = k_or_rank ? k_or_rank[l] : L.cap;
    return (k >= 1 && k <= L.cap) ? k : 0;  // out of range: the layer contributes nothing
}

// bounds[w][L.dc_base + tt] = first payload entry of (w, l) whose index lies in
// decode tile tt or later; slot ntiles holds k.
__global__ void __launch_bounds__(256) dc_bounds_kernel(const DevLayer* __restrict__ layers,
                                                        const int32_t* __restrict__ bunit_layer,
                                                        const int32_t* __restrict__ bunit_chunk,
                                                        int32_t bunits_pw, int32_t W,
                                                        int64_t vals_pw, int32_t dc_slots,
                                                        const int32_t* __restrict__ k_or_rank,
                                                        const int32_t* __restrict__ idx,
                                                        int32_t* __restrict__ bounds) {
    const int64_t total = int64_t(bunits_pw) * W;
    for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
        const int w = int(u / bunits_pw);
        const int bu = int(u % bunits_pw);
        const int32_t l = bunit_layer[bu];
        const DevLayer L = layers[l];
        const int32_t k = layer_k(L, k_or_rank, l);
        int32_t* b = bounds + int64_t(w) * dc_slots + L.dc_base;
        const int32_t nt = L.dc_ntiles;
        const int64_t j0 = int64_t(bunit_chunk[bu]) * kDcBoundChunk;
        if (k == 0) {
            if (j0 == 0)
                for (int32_t tt = threadIdx.x; tt <= nt; tt += blockDim.x) b[tt] = 0;
            continue;
        }
        const int32_t* ix = idx + int64_t(w) * vals_pw + L.val_off;
        const int64_t j1 = min64(j0 + kDcBoundChunk, k);
        for (int64_t j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
            const int32_t tj = min(max(ix[j], 0) >> kDcTileLog, nt);
            const int32_t tp = j > 0 ? min(max(ix[j - 1], 0) >> kDcTileLog, nt) : -1;
            for (int32_t tt = tp + 1; tt <= tj; ++tt) b[tt] = int32_t(j);
            if (j == k - 1)
                for (int32_t tt = tj + 1; tt <= nt; ++tt) b[tt] = k;
        }
    }
}

__global__ void __launch_bounds__(256) dc_accum_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ dc_tile_layer,
    const int32_t* __restrict__ tile_list, int32_t dc_tiles, int32_t W, int64_t vals_pw,
    int64_t P_pw, int64_t Q_pw, int32_t dc_slots, const int32_t* __restrict__ k_or_rank,
    const float* __restrict__ vals, const int32_t* __restrict__ idx, const float* __restrict__ P,
    const float* __restrict__ Q, const int32_t* __restrict__ bounds, float scale,
    float* __restrict__ out) {
    __shared__ __align__(16) float acc[kDcTile];
    __shared__ int32_t s_first[32], s_off[33];
    __shared__ int32_t s_sidx[kDcStage];
    __shared__ float s_sval[kDcStage];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
            for (int i = threadIdx.x; i < kDcTile / 4; i += blockDim.x)
                reinterpret_cast<float4*>(acc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            // every worker's entry range for this tile at once, then one staged
            // load of all the entries, so the worker-order sums below touch
            // only shared memory
            if (W <= 32 && warp == 0) {
                int32_t a = 0, e = 0;
                if (lane < W) {
                    const int32_t* b = bounds + int64_t(lane) * dc_slots + L.dc_base + tt;
                    a = min(max(b[0], 0), k);
                    e = min(max(b[1], a), k);
                    s_first[lane] = a;
                }
                const int c = e - a;
                const int incl = warp_inclusive_scan(c);
                if (lane < W) s_off[lane] = incl - c;
                if (lane == 31) s_off[32] = incl;
            }
            __syncthreads();
            const bool staged = W <= 32 && s_off[32] <= kDcStage;
            if (staged) {
                const int total = s_off[32];
                for (int q = threadIdx.x; q < total; q += blockDim.x) {
                    int w = 0;
                    while (w + 1 < W && s_off[w + 1] <= q) ++w;
                    const int64_t j = int64_t(s_first[w]) + (q - s_off[w]);
                    const int64_t o2 = int64_t(w) * vals_pw + L.val_off + j;
                    s_sidx[q] = int32_t(int64_t(idx[o2]) - start);
                    s_sval[q] = vals[o2];
                }
                for (int w = 0; w < W; ++w) {
                    __syncthreads();
                    for (int q = s_off[w] + threadIdx.x; q < s_off[w + 1 < W ? w + 1 : 32];
                         q += blockDim.x) {
                        const int i = s_sidx[q];
                        if (i >= 0 && i < cnt) acc[i] = __fadd_rn(acc[i], s_sval[q]);
                    }
                }
            } else {
                for (int w = 0; w < W; ++w) {
                    __syncthreads();
                    const int32_t* b = bounds + int64_t(w) * dc_slots + L.dc_base + tt;
                    const int32_t a = min(max(b[0], 0), k), e = min(max(b[1], a), k);
                    const float* v = vals + int64_t(w) * vals_pw + L.val_off;
                    const int32_t* ix = idx + int64_t(w) * vals_pw + L.val_off;
                    for (int32_t j = a + threadIdx.x; j < e; j += blockDim.x) {
                        const int64_t i = int64_t(ix[j]) - start;
                        if (i >= 0 && i < cnt) acc[i] = __fadd_rn(acc[i], v[j]);
                    }
                }
            }
            __syncthreads();
            if (cnt == kDcTile && ((L.offset + start) & 3) == 0) {
                for (int i = threadIdx.x; i < kDcTile / 4; i += blockDim.x) {
                    const float4 a = reinterpret_cast<const float4*>(acc)[i];
                    reinterpret_cast<float4*>(o)[i] =
                        make_float4(__fmul_rn(a.x, scale), __fmul_rn(a.y, scale),
                                    __fmul_rn(a.z, scale), __fmul_rn(a.w, scale));
                }
            } else {
                for (int i = threadIdx.x; i < cnt; i += blockDim.x) o[i] = __fmul_rn(acc[i], scale);
            }
            __syncthreads();
        } else if (L.kind == GCE_KIND_DENSE) {
            for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
                float s = 0.0f;
                for (int w = 0; w < W; ++w)
                    s = __fadd_rn(s, vals[int64_t(w) * vals_pw + L.val_off + start + i]);
                o[i] = __fmul_rn(s, scale);
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
                o[i] = __fmul_rn(s, scale);
                col += blockDim.x;
                if (col >= cols) {
                    row += col / cols;
                    col %= cols;
                }
            }
        }
    }
}

// bounds pass plus the decode kernels for every kind the table holds
static int launch_decode(const gce_table* t, int32_t W, const float* vals, const int32_t* idx,
                         const int32_t* k_or_rank, const float* P, const float* Q, float scale,
                         float* out, int32_t* bounds, cudaStream_t st) {
    const bool sparse = t->ckind == GCE_KIND_TOPK || t->ckind == GCE_KIND_RANDK;
    const int sms = sm_count();
    if (sparse && t->bunits_pw > 0) {
        const int64_t units = int64_t(t->bunits_pw) * W;
        GCE_LAUNCH(dc_bounds_kernel, int(min64(units, int64_t(sms) * 8)), 256, 0, st, t->d_layers,
                   t->d_bunit_layer, t->d_bunit_chunk, t->bunits_pw, W, t->vals_pw, t->dc_slots,
                   k_or_rank, idx, bounds);
    }
    if (t->nps > 0 && launch_lowrank_decode(t, W, k_or_rank, P, Q, scale, out, st)) {
        // PowerSGD layers done by their own tiled kernel; the rest here
        if (t->dc_nl_n > 0)
            GCE_LAUNCH(dc_accum_kernel, int(min64(t->dc_nl_n, int64_t(sms) * 8)), 256, 0, st,
                       t->d_layers, t->d_dc_tile_layer, t->d_dc_nl_tiles, t->dc_nl_n, W,
                       t->vals_pw, t->P_pw, t->Q_pw, t->dc_slots, k_or_rank, vals, idx, P, Q,
                       bounds, scale, out);
        return check_launch();
    }
    GCE_LAUNCH(dc_accum_kernel, int(min64(t->dc_tiles, int64_t(sms) * 8)), 256, 0, st,
               t->d_layers, t->d_dc_tile_layer, nullptr, t->dc_tiles, W, t->vals_pw, t->P_pw,
               t->Q_pw, t->dc_slots, k_or_rank, vals, idx, P, Q, bounds, scale, out);
    return check_launch();
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

// ---- decode without a caller workspace -------------------------------------------------
// Some callers cannot hand the library a workspace: code that runs inside
// another allocator (a caching allocator's out-of-memory hook, for one), code
// whose device memory is all reserved up front by its framework, and code in
// a latency-critical loop that must not pay cudaMalloc's implicit device-wide
// synchronisation.  For them, decompress_accumulate_noalloc keeps its only
// scratch -- the per-tile entry bounds -- in the fixed array below, which the
// module reserves on every GPU that loads this library until the process
// exits.  4 MiB: W x (decode tiles of 4096 elements + layers) <= 1,048,576
// bound slots (the BERT-base table at W = 8 uses 214,144).
constexpr int64_t kNoAllocBoundSlots = int64_t(1) << 20;
static __device__ __align__(256) int32_t g_noalloc_bounds[kNoAllocBoundSlots];

// Device address of g_noalloc_bounds on the current device, looked up once per
// device (host code cannot use the symbol itself as a device address).
static int32_t* noalloc_bounds_on_current_device() {
    static std::mutex mu;
    static int32_t* addr[64] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_bounds) != cudaSuccess || !p) return nullptr;
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
    int32_t* bounds = noalloc_bounds_on_current_device();
    if (!bounds) return GCE_ERR_CUDA;
    // every bound slot a sparse layer uses is rewritten by the bounds pass, so
    // nothing left from an earlier call needs clearing
    return launch_decode(t, W, vals, idx, k_or_rank, P, Q, scale, out, bounds,
                         static_cast<cudaStream_t>(stream));
}
