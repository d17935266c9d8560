// accordion.cu -- Accordion's per-layer critical-regime detector on sm_100a.
//
// "Accordion: Adaptive Gradient Communication via Critical Learning Regime
// Identification", Method: the rate of change of each layer's gradient norm
// marks critical regimes; inside one the layer uses the low-compression
// level l_low (higher rank / larger k), outside it the high-compression level
// l_high.  On a check step (step % interval == 0) every compressed layer's
// norm s = sqrt(sum g^2) is taken (fp32 in, fp64 accumulation in a fixed
// order) and compared with the previous check's:
//   rel = |s_prev - s| / s_prev  (s_prev == 0: 0 if s == 0, else +inf)
//   level = (no previous check or rel >= threshold) ? LOW : HIGH.
// Every step then maps the level to k (parts per million of the layer,
// k = max(1, floor(n * ppm / 1e6))) or to the rank.
//
// Kernels: norm (one pass over the gradient, 4 B per element, per-tile fp64
// partials) and decide (one warp per layer: tile partials in a fixed lane /
// tree order, then the decision); on other steps only levels -> k / rank.
#include <cmath>

#include "common.cuh"
#include "scan.cuh"

namespace gce {

constexpr int kAcTile = 16384;  // gradient elements per norm tile

int accordion_plan(gce_table* t) {
    std::vector<int2> tiles, per(t->L, make_int2(0, 0));
    for (int32_t l = 0; l < t->L; ++l) {
        const DevLayer& L = t->layers[l];
        if (L.kind == GCE_KIND_DENSE) continue;
        const int32_t nt = int32_t((L.n + kAcTile - 1) / kAcTile);
        per[l] = make_int2(int32_t(tiles.size()), nt);
        for (int32_t c = 0; c < nt; ++c) tiles.push_back(make_int2(l, c));
    }
    t->ac_ntiles = int32_t(tiles.size());
    t->d_ac_tiles = nullptr;
    t->d_ac_layer = nullptr;
    if (cudaMalloc(&t->d_ac_layer, per.size() * sizeof(int2)) != cudaSuccess) return GCE_ERR_NOMEM;
    if (cudaMemcpy(t->d_ac_layer, per.data(), per.size() * sizeof(int2), cudaMemcpyHostToDevice) !=
        cudaSuccess)
        return GCE_ERR_CUDA;
    if (!tiles.empty()) {
        if (cudaMalloc(&t->d_ac_tiles, tiles.size() * sizeof(int2)) != cudaSuccess) return GCE_ERR_NOMEM;
        if (cudaMemcpy(t->d_ac_tiles, tiles.data(), tiles.size() * sizeof(int2),
                       cudaMemcpyHostToDevice) != cudaSuccess)
            return GCE_ERR_CUDA;
    }
    return GCE_OK;
}

void accordion_plan_free(gce_table* t) {
    cudaFree(t->d_ac_tiles);
    cudaFree(t->d_ac_layer);
}

size_t accordion_ws_bytes(const gce_table* t) {
    Carver c;
    c.take<double>(t->ac_ntiles);
    return c.off;
}

__global__ void __launch_bounds__(256) ac_norm_kernel(const DevLayer* __restrict__ layers,
                                                      const int2* __restrict__ tiles, int32_t ntiles,
                                                      const float* __restrict__ grad,
                                                      double* __restrict__ part) {
    grid_dependency_sync();
    __shared__ double s_red[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int32_t u = blockIdx.x; u < ntiles; u += gridDim.x) {
        const int2 d = tiles[u];
        const DevLayer L = layers[d.x];
        const int64_t start = int64_t(d.y) * kAcTile;
        const int cnt = int(min64(kAcTile, L.n - start));
        const float* g = grad + L.offset + start;
        double s = 0.0;
        if (((L.offset + start) & 3) == 0) {
            const int c4 = cnt >> 2;
            for (int i = tid; i < c4; i += blockDim.x) {
                const float4 x = ld_stream4(g + 4 * i);
                s = fma(double(x.x), double(x.x), s);
                s = fma(double(x.y), double(x.y), s);
                s = fma(double(x.z), double(x.z), s);
                s = fma(double(x.w), double(x.w), s);
            }
            for (int i = 4 * c4 + tid; i < cnt; i += blockDim.x) s = fma(double(g[i]), double(g[i]), s);
        } else {
            for (int i = tid; i < cnt; i += blockDim.x) s = fma(double(g[i]), double(g[i]), s);
        }
        s = warp_sum(s);
        if (lane == 0) s_red[warp] = s;
        __syncthreads();
        if (tid == 0) {
            double t = 0.0;
            for (int i = 0; i < 8; ++i) t += s_red[i];
            part[u] = t;
        }
        __syncthreads();
    }
}

__device__ __forceinline__ int32_t ac_param(const DevLayer& L, int32_t level, int32_t lvl_low,
                                            int32_t lvl_high) {
    const int32_t p = level == GCE_LEVEL_LOW ? lvl_low : lvl_high;
    if (L.kind == GCE_KIND_POWERSGD) return p;
    if (L.kind == GCE_KIND_SIGN) return 0;  // one fixed level: nothing to choose
    const int64_t k = (L.n * int64_t(p)) / 1000000;
    return int32_t(k < 1 ? 1 : k);
}

// A layer's sum of squares from its tile partials, in a fixed order: lane i
// adds tiles i, i + 32, ... in order, then the lanes' sums by warp_sum.  Run by
// a full warp.
__device__ __forceinline__ double ac_layer_sumsq(const int2 pl, const double* __restrict__ part) {
    const int lane = threadIdx.x & 31;
    double s = 0.0;
    for (int i = lane; i < pl.y; i += 32) s += part[pl.x + i];
    return warp_sum(s);
}

// one warp per layer: sumsq[l] (0 for DENSE layers)
__global__ void __launch_bounds__(256) ac_sumsq_kernel(const DevLayer* __restrict__ layers,
                                                       const int2* __restrict__ ac_layer, int32_t L,
                                                       const double* __restrict__ part,
                                                       double* __restrict__ sumsq) {
    grid_dependency_sync();
    const int lane = threadIdx.x & 31;
    const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t l = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); l < L; l += wstride) {
        const double s = layers[l].kind == GCE_KIND_DENSE ? 0.0 : ac_layer_sumsq(ac_layer[l], part);
        if (lane == 0) sumsq[l] = s;
    }
}

// one warp per layer; the sums of squares from the tile partials, or (sumsq
// non-null) given per layer
__global__ void __launch_bounds__(256) ac_decide_kernel(
    const DevLayer* __restrict__ layers, const int2* __restrict__ ac_layer, int32_t L,
    const double* __restrict__ part, const double* __restrict__ sumsq, int32_t check,
    double threshold, int32_t lvl_low, int32_t lvl_high, double* __restrict__ prev_norm,
    int32_t* __restrict__ level, double* __restrict__ cur_norm, int32_t* __restrict__ k_or_rank) {
    grid_dependency_sync();
    const int lane = threadIdx.x & 31;
    const int64_t wstride = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t l = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); l < L; l += wstride) {
        const DevLayer Ld = layers[l];
        if (Ld.kind == GCE_KIND_DENSE) {
            if (lane == 0) k_or_rank[l] = 0;
            continue;
        }
        int32_t lv = level[l];
        if (check) {
            const double s = sumsq ? sumsq[l] : ac_layer_sumsq(ac_layer[l], part);
            const double cur = sqrt(s);
            const double prev = prev_norm[l];
            double rel;
            if (prev < 0.0) {
                rel = INFINITY;
            } else if (prev == 0.0) {
                rel = cur == 0.0 ? 0.0 : INFINITY;
            } else {
                rel = fabs(prev - cur) / prev;
            }
            lv = (prev < 0.0 || rel >= threshold) ? GCE_LEVEL_LOW : GCE_LEVEL_HIGH;
            if (lane == 0) {
                level[l] = lv;
                prev_norm[l] = cur;
                if (cur_norm) cur_norm[l] = cur;
            }
        }
        if (lane == 0) k_or_rank[l] = ac_param(Ld, lv, lvl_low, lvl_high);
    }
}

__global__ void ac_init_kernel(int32_t L, double* __restrict__ prev_norm, int32_t* __restrict__ level) {
    grid_dependency_sync();
    for (int32_t l = blockIdx.x * blockDim.x + threadIdx.x; l < L; l += gridDim.x * blockDim.x) {
        prev_norm[l] = -1.0;
        level[l] = GCE_LEVEL_LOW;
    }
}

}  // namespace gce

using namespace gce;

extern "C" int accordion_init(const gce_table* t, double* prev_norm, int32_t* level, void* stream) {
    if (!t || !prev_norm || !level) return GCE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    GCE_LAUNCH(ac_init_kernel, (t->L + 255) / 256, 256, 0, st, t->L, prev_norm, level);
    return check_launch();
}

extern "C" int accordion_select(const gce_table* t, const float* grad, int64_t step,
                                int32_t interval, double threshold, int32_t lvl_low,
                                int32_t lvl_high, double* prev_norm, int32_t* level,
                                double* cur_norm, int32_t* k_or_rank_out, void* ws,
                                size_t ws_bytes, void* stream) {
    if (!t || !grad || !prev_norm || !level || !k_or_rank_out || !ws) return GCE_ERR_ARG;
    if (interval < 1 || step < 0 || !(threshold >= 0.0)) return GCE_ERR_ARG;
    if (!aligned16(grad) || !aligned16(ws)) return GCE_ERR_ARG;
    if (t->ckind == GCE_KIND_POWERSGD) {
        if (lvl_low < 1 || lvl_low > kMaxRank || lvl_high < 1 || lvl_high > kMaxRank) return GCE_ERR_ARG;
    } else if (lvl_low < 1 || lvl_low > 1000000 || lvl_high < 1 || lvl_high > 1000000) {
        return GCE_ERR_ARG;
    }
    if (ws_bytes < accordion_ws_bytes(t)) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    double* part = at<double>(ws, GCE_WS_HEADER_BYTES);
    const int check = (step % interval) == 0;
    static const int r_norm = resident_blocks(ac_norm_kernel, 256);
    static const int r_decide = resident_blocks(ac_decide_kernel, 256);
    if (check && t->ac_ntiles > 0)
        GCE_LAUNCH(ac_norm_kernel, wave_grid(t->ac_ntiles, 8, r_norm), 256, 0, st,
                   t->d_layers, t->d_ac_tiles, t->ac_ntiles, grad, part);
    GCE_LAUNCH(ac_decide_kernel, wave_grid((t->L + 7) / 8, 4, r_decide), 256, 0, st,
               t->d_layers, t->d_ac_layer, t->L, part, nullptr, check, threshold, lvl_low,
               lvl_high, prev_norm, level, cur_norm, k_or_rank_out);
    return check_launch();
}

extern "C" int accordion_sumsq(const gce_table* t, const float* grad, double* sumsq, void* ws,
                               size_t ws_bytes, void* stream) {
    if (!t || !grad || !sumsq || !ws || !aligned16(grad) || !aligned16(ws)) return GCE_ERR_ARG;
    if (ws_bytes < accordion_ws_bytes(t)) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    double* part = at<double>(ws, GCE_WS_HEADER_BYTES);
    static const int r_norm = resident_blocks(ac_norm_kernel, 256);
    static const int r_sum = resident_blocks(ac_sumsq_kernel, 256);
    if (t->ac_ntiles > 0)
        GCE_LAUNCH(ac_norm_kernel, wave_grid(t->ac_ntiles, 8, r_norm), 256, 0, st,
                   t->d_layers, t->d_ac_tiles, t->ac_ntiles, grad, part);
    GCE_LAUNCH(ac_sumsq_kernel, wave_grid((t->L + 7) / 8, 4, r_sum), 256, 0, st, t->d_layers,
               t->d_ac_layer, t->L, part, sumsq);
    return check_launch();
}

extern "C" int accordion_decide(const gce_table* t, const double* sumsq, int64_t step,
                                int32_t interval, double threshold, int32_t lvl_low,
                                int32_t lvl_high, double* prev_norm, int32_t* level,
                                double* cur_norm, int32_t* k_or_rank_out, void* stream) {
    if (!t || !prev_norm || !level || !k_or_rank_out) return GCE_ERR_ARG;
    if (interval < 1 || step < 0 || !(threshold >= 0.0)) return GCE_ERR_ARG;
    if (t->ckind == GCE_KIND_POWERSGD) {
        if (lvl_low < 1 || lvl_low > kMaxRank || lvl_high < 1 || lvl_high > kMaxRank) return GCE_ERR_ARG;
    } else if (lvl_low < 1 || lvl_low > 1000000 || lvl_high < 1 || lvl_high > 1000000) {
        return GCE_ERR_ARG;
    }
    const int check = (step % interval) == 0;
    if (check && !sumsq) return GCE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    static const int r_decide = resident_blocks(ac_decide_kernel, 256);
    GCE_LAUNCH(ac_decide_kernel, wave_grid((t->L + 7) / 8, 4, r_decide), 256, 0, st,
               t->d_layers, t->d_ac_layer, t->L, nullptr, sumsq, check, threshold, lvl_low,
               lvl_high, prev_norm, level, cur_norm, k_or_rank_out);
    return check_launch();
}
