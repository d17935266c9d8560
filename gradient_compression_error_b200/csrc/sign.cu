// sign.cu -- signSGD with error feedback on sm_100a.
//
// "On the Utility of Gradient Compression in Distributed Training Systems",
// Method / Key results: sign SGD sends one bit per element and, having no
// all-reduce, is gathered.  "Sparsified SGD with Memory", Method: the memory
// keeps what the compressed update leaves out.  Per (worker, SIGN layer):
//   p = fl(m + fl(eta*g));  s = fl(sum |p| / n), the sum in fp64;
//   payload: s and the sign bits of p;  m <- fl(p - s) or fl(p + s).
//
// Two passes over grad and mem (8 B/element, then 12 B/element plus 1/8 B
// of sign words): the scale needs the whole layer before the first element
// can be updated.
//   norm   per 8192-element tile an fp64 partial of |p| (fixed reduction
//          order); the block that finishes a layer's last tile adds the
//          layer's partials (strided over its threads, then a fixed tree)
//          and writes s
//   emit   p again, the memory update and the packed sign words: each lane
//          holds four neighbouring elements, eight lanes form one 32-bit word
// The aggregates live in decompress.cu (worker-order sum) and here (the
// majority vote).
#include "common.cuh"
#include "scan.cuh"
#include "topk_layout.cuh"

namespace gce {

struct SgLayout {
    size_t partials = 0, done = 0, scales = 0, total = 0;
};

static SgLayout sg_layout(const gce_table* t, int32_t W) {
    SgLayout o;
    Carver c;
    const bool on = t->ckind == GCE_KIND_SIGN;
    o.partials = c.take<double>(on ? int64_t(W) * t->tiles_pw : 0);
    o.done = c.take<int32_t>(on ? int64_t(W) * int64_t(t->comp.size()) : 0);
    o.scales = c.take<float>(on ? int64_t(W) * int64_t(t->comp.size()) : 0);
    o.total = c.off;
    return o;
}

size_t sign_ws_bytes(const gce_table* t, int32_t W) { return sg_layout(t, W).total; }

__device__ __forceinline__ double block_sum_fixed(double x, double* s_red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    x = warp_sum(x);
    if (lane == 0) s_red[warp] = x;
    __syncthreads();
    double t = 0.0;
    for (int i = 0; i < int(blockDim.x >> 5); ++i) t += s_red[i];
    __syncthreads();
    return t;
}

// ---- pass 1: the layer scale -------------------------------------------------------
__global__ void __launch_bounds__(256) sg_norm_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t W, int32_t ncomp, int64_t N, int64_t vals_pw, const float* __restrict__ grad,
    const float* __restrict__ mem, float eta, double* __restrict__ partials,
    int32_t* __restrict__ done, float* __restrict__ scales, float* __restrict__ vals,
    int32_t* __restrict__ status) {
    __shared__ double s_red[8];
    __shared__ int s_last;
    const int tid = threadIdx.x;
    for (int64_t t = blockIdx.x; t < int64_t(tiles_pw) * W; t += gridDim.x) {
        const int w = int(t / tiles_pw);
        const int lt = int(t % tiles_pw);
        const DevLayer L = layers[tile_layer[lt]];
        const int64_t s0 = int64_t(lt - L.tile0) * kTkTile;
        const int cnt = int(min64(kTkTile, L.n - s0));
        const int64_t base = int64_t(w) * N + L.offset + s0;
        double acc = 0.0;
        if ((base & 3) == 0 && cnt == kTkTile) {
#pragma unroll
            for (int q = 0; q < kTkTile / 4 / 256; ++q) {
                const int e = 4 * (q * 256 + tid);
                const float4 g = ld_stream4(grad + base + e);
                const float4 m = *reinterpret_cast<const float4*>(mem + base + e);
                acc += fabs(double(residual(m.x, eta, g.x))) + fabs(double(residual(m.y, eta, g.y))) +
                       fabs(double(residual(m.z, eta, g.z))) + fabs(double(residual(m.w, eta, g.w)));
            }
        } else {
            for (int e = tid; e < cnt; e += 256)
                acc += fabs(double(residual(mem[base + e], eta, grad[base + e])));
        }
        // a NaN or infinite p makes the sum non-finite
        flag_nonfinite(!(fabs(acc) < 1.0e308), status);
        acc = block_sum_fixed(acc, s_red);
        if (tid == 0) {
            partials[t] = acc;
            __threadfence();
            s_last = atomicAdd(&done[int64_t(w) * ncomp + L.sidx], 1) == L.ntiles - 1;
        }
        __syncthreads();
        if (s_last) {  // the whole block adds the layer's partials (fixed order)
            __threadfence();
            const double* pp = partials + int64_t(w) * tiles_pw + L.tile0;
            double part = 0.0;
            for (int i = tid; i < L.ntiles; i += blockDim.x) part += __ldcg(pp + i);
            const double sum = block_sum_fixed(part, s_red);
            if (tid == 0) {
                const float s = float(sum / double(L.n));
                scales[int64_t(w) * ncomp + L.sidx] = s;
                float* slot = vals + int64_t(w) * vals_pw + L.val_off;
                slot[0] = s;
                slot[1] = slot[2] = slot[3] = 0.0f;
            }
        }
        __syncthreads();
    }
}

// ---- pass 2: memory update and sign words -------------------------------------------
__device__ __forceinline__ float sg_update(float p, float s, uint32_t& neg) {
    neg = __float_as_uint(p) >> 31;
    return neg ? __fadd_rn(p, s) : __fsub_rn(p, s);
}

__global__ void __launch_bounds__(256) sg_emit_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t W, int32_t ncomp, int64_t N, int64_t vals_pw, const float* __restrict__ grad,
    float* __restrict__ mem, float eta, const float* __restrict__ scales,
    float* __restrict__ vals) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t t = blockIdx.x; t < int64_t(tiles_pw) * W; t += gridDim.x) {
        const int w = int(t / tiles_pw);
        const int lt = int(t % tiles_pw);
        const DevLayer L = layers[tile_layer[lt]];
        const int64_t s0 = int64_t(lt - L.tile0) * kTkTile;
        const int cnt = int(min64(kTkTile, L.n - s0));
        const int64_t base = int64_t(w) * N + L.offset + s0;
        const float s = scales[int64_t(w) * ncomp + L.sidx];
        uint32_t* words =
            reinterpret_cast<uint32_t*>(vals + int64_t(w) * vals_pw + L.val_off + 4) + s0 / 32;
        const int e0 = warp * (kTkTile / 8);  // this warp's 1024 elements
        if ((base & 3) == 0 && cnt == kTkTile) {
            // all loads of the warp's 1024 elements first, then the updates
            float4 g[8], m[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int e = e0 + 128 * q + 4 * lane;
                g[q] = ld_stream4(grad + base + e);
                m[q] = *reinterpret_cast<const float4*>(mem + base + e);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int e = e0 + 128 * q + 4 * lane;
                uint32_t n0, n1, n2, n3;
                float4 r;
                r.x = sg_update(residual(m[q].x, eta, g[q].x), s, n0);
                r.y = sg_update(residual(m[q].y, eta, g[q].y), s, n1);
                r.z = sg_update(residual(m[q].z, eta, g[q].z), s, n2);
                r.w = sg_update(residual(m[q].w, eta, g[q].w), s, n3);
                __stcs(reinterpret_cast<float4*>(mem + base + e), r);
                // eight lanes hold one word's 32 bits, four each
                uint32_t v = (n0 | (n1 << 1) | (n2 << 2) | (n3 << 3)) << (4 * (lane & 7));
                v |= __shfl_xor_sync(kFull, v, 1);
                v |= __shfl_xor_sync(kFull, v, 2);
                v |= __shfl_xor_sync(kFull, v, 4);
                if ((lane & 7) == 0) words[(e0 + 128 * q) / 32 + (lane >> 3)] = v;
            }
        } else {
            // ragged or unaligned tile: one element a lane, a ballot a word
            for (int q = 0; q < kTkTile / 8 / 32; ++q) {
                const int e = e0 + 32 * q + lane;
                uint32_t neg = 0;
                if (e < cnt) mem[base + e] = sg_update(residual(mem[base + e], eta, grad[base + e]), s, neg);
                const uint32_t word = __ballot_sync(kFull, neg != 0);
                if (lane == 0 && e0 + 32 * q < cnt) words[(e0 + 32 * q) / 32] = word;
            }
        }
    }
}

// ---- majority vote ---------------------------------------------------------------------
__global__ void __launch_bounds__(128) sg_vote_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ dc_tile_layer,
    int32_t dc_tiles, int32_t W, int64_t vals_pw, const float* __restrict__ vals, float scale,
    float* __restrict__ out) {
    for (int32_t u = blockIdx.x; u < dc_tiles; u += gridDim.x) {
        const int32_t l = dc_tile_layer[u];
        const DevLayer L = layers[l];
        const int64_t start = int64_t(u - L.dc_tile0) << kDcTileLog;
        const int cnt = int(min64(kDcTile, L.n - start));
        float* o = out + L.offset + start;
        if (L.kind == GCE_KIND_SIGN) {
            for (int i = 4 * int(threadIdx.x); i < cnt; i += 4 * int(blockDim.x)) {
                int c[4] = {0, 0, 0, 0};
                // eight workers' words in flight at a time
                for (int w0 = 0; w0 < W; w0 += 8) {
                    uint32_t nib[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        nib[e] = 0u;
                        if (w0 + e < W)
                            nib[e] = reinterpret_cast<const uint32_t*>(
                                vals + int64_t(w0 + e) * vals_pw + L.val_off + 4)[(start + i) >> 5] >>
                                ((start + i) & 31);
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (w0 + e < W)
#pragma unroll
                            for (int j = 0; j < 4; ++j) c[j] += ((nib[e] >> j) & 1u) ? -1 : 1;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (i + j < cnt) o[i + j] = c[j] > 0 ? scale : (c[j] < 0 ? -scale : 0.0f);
            }
        } else if (L.kind == GCE_KIND_DENSE) {
            for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
                float s = 0.0f;
                for (int w = 0; w < W; ++w)
                    s = __fadd_rn(s, vals[int64_t(w) * vals_pw + L.val_off + start + i]);
                o[i] = __fmul_rn(s, scale);
            }
        }
    }
}

}  // namespace gce

using namespace gce;

extern "C" int ef_sign_step(const gce_table* t, int32_t W, const float* grad, float* mem,
                            float eta, float* vals, void* ws, size_t ws_bytes, void* stream) {
    if (!t || W < 1 || !grad || !mem || !ws) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_SIGN && t->ckind != -1) return GCE_ERR_KIND;
    if (!aligned16(grad) || !aligned16(mem) || !aligned16(ws)) return GCE_ERR_ARG;
    if (t->vals_pw > 0 && (!vals || !aligned16(vals))) return GCE_ERR_ARG;
    const SgLayout lay = sg_layout(t, W);
    if (ws_bytes < lay.total) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = static_cast<int32_t*>(ws);
    if (t->ckind == GCE_KIND_SIGN && t->tiles_pw > 0) {
        const int32_t ncomp = int32_t(t->comp.size());
        int32_t* done = at<int32_t>(ws, lay.done);
        if (cudaMemsetAsync(done, 0, sizeof(int32_t) * size_t(W) * ncomp, st) != cudaSuccess)
            return GCE_ERR_CUDA;
        static const int r_norm = resident_blocks(sg_norm_kernel, 256);
        static const int r_emit = resident_blocks(sg_emit_kernel, 256);
        const int64_t tiles = int64_t(t->tiles_pw) * W;
        GCE_LAUNCH(sg_norm_kernel, wave_grid(tiles, 8, r_norm), 256, 0, st, t->d_layers,
                   t->d_tile_layer, t->tiles_pw, W, ncomp, t->N, t->vals_pw, grad, mem, eta,
                   at<double>(ws, lay.partials), done, at<float>(ws, lay.scales), vals,
                   status);
        GCE_LAUNCH(sg_emit_kernel, wave_grid(tiles, 8, r_emit), 256, 0, st, t->d_layers,
                   t->d_tile_layer, t->tiles_pw, W, ncomp, t->N, t->vals_pw, grad, mem, eta,
                   at<float>(ws, lay.scales), vals);
        if (check_launch() != GCE_OK) return GCE_ERR_CUDA;
    }
    return launch_dense_layers(t, W, grad, mem, eta, vals, status, st);
}

extern "C" int decompress_vote(const gce_table* t, int32_t W, const float* vals, float scale,
                               float* out, void* stream) {
    if (!t || W < 1 || !out || !aligned16(out)) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_SIGN && t->ckind != -1) return GCE_ERR_KIND;
    if (t->vals_pw > 0 && !vals) return GCE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    static const int r_vote = resident_blocks(sg_vote_kernel, 128);
    if (t->dc_tiles > 0)
        GCE_LAUNCH(sg_vote_kernel, wave_grid(t->dc_tiles, 16, r_vote), 128, 0, st, t->d_layers,
                   t->d_dc_tile_layer, t->dc_tiles, W, t->vals_pw, vals, scale, out);
    return check_launch();
}
