// sign.cu -- signSGD with error feedback on sm_100a.
//
// "On the Utility of Gradient Compression in Distributed Training Systems",
// Method / Key results: sign SGD sends one bit per element and, having no
// all-reduce, is gathered.  "Sparsified SGD with Memory", Method: the memory
// keeps what the compressed update leaves out.  Per (worker, SIGN layer):
//   p = fl(m + fl(eta*g));  s = fl(sum |p| / n), the sum in fp64;
//   payload: s and the sign bits of p;  m <- fl(p - s) or fl(p + s).
//
// The scale needs the whole layer before the first element can be updated,
// so every element is visited twice:
//   norm   per 8192-element tile an fp64 partial of |p| (fixed reduction
//          order); the block that finishes a layer's last tile adds the
//          layer's partials (strided over its threads, then a fixed tree)
//          and writes s
//   emit   p again, the memory update and the packed sign words: each lane
//          holds four neighbouring elements, eight lanes form one 32-bit word
// Two ways to schedule the visits:
//   pipelined (sg_fused_kernel, one launch): norm tiles run a bounded
//          distance ahead of emit tiles, so an emit tile's grad and memory
//          are still in L2 and HBM sees them once (8 B/element read, 4 B
//          written, plus 1/8 B of sign words).  The norm reads with an L2
//          evict-last policy and the emit re-reads with evict-first, so
//          the lines wait in L2 for their second visit and leave after it;
//   two passes (sg_norm_kernel, then sg_emit_kernel): 8 B/element, then
//          12 B/element; used while a stream is being captured before the
//          pipelined schedule exists, or when it is switched off.
// Both give the same bits: the partials, their order and the scale are the
// same.  The aggregates live in decompress.cu (worker-order sum) and here
// (the majority vote).
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "scan.cuh"
#include "topk_layout.cuh"

namespace gce {

// Workspace: per-tile partials; the per-(worker, layer) sync words (tiles
// done, then scale ready) and the work counter of the pipelined kernel,
// cleared by one memset; the scales.
struct SgLayout {
    size_t partials = 0, sync = 0, scales = 0, total = 0;
};

static SgLayout sg_layout(const gce_table* t, int32_t W) {
    SgLayout o;
    Carver c;
    const bool on = t->ckind == GCE_KIND_SIGN;
    const int64_t segs = int64_t(W) * int64_t(t->comp.size());
    o.partials = c.take<double>(on ? int64_t(W) * t->tiles_pw : 0);
    o.sync = c.take<int32_t>(on ? 2 * segs + 1 : 0);
    o.scales = c.take<float>(on ? segs : 0);
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

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ float4 ld_hint4(const float* p, uint64_t pol) {
    float4 v;
    asm volatile("ld.global.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

// Where tile t (worker-major over the compressed layers) lies.
struct SgTile {
    DevLayer L;
    int64_t s0, base, seg;
    int w, cnt;
};

__device__ __forceinline__ SgTile sg_tile(const DevLayer* layers, const int32_t* tile_layer,
                                          int32_t tiles_pw, int32_t ncomp, int64_t N, int64_t t) {
    SgTile x;
    x.w = int(t / tiles_pw);
    const int lt = int(t % tiles_pw);
    x.L = layers[tile_layer[lt]];
    x.s0 = int64_t(lt - x.L.tile0) * kTkTile;
    x.cnt = int(min64(kTkTile, x.L.n - x.s0));
    x.base = int64_t(x.w) * N + x.L.offset + x.s0;
    x.seg = int64_t(x.w) * ncomp + x.L.sidx;
    return x;
}

// ---- norm of one tile ---------------------------------------------------------------
// The tile's fp64 partial of |p|; the block that completes the layer adds
// the layer's partials in a fixed order, writes s (scales and the payload
// slot) and, when `ready` is given, publishes it.  kKeep: L2 evict-last
// loads, so the lines stay for the emit that follows; otherwise grad is read
// evict-first.  Ends with the block synchronised.
template <bool kKeep>
__device__ __forceinline__ void sg_norm_tile(const SgTile& x, int64_t t, int32_t tiles_pw,
                                             int64_t vals_pw, const float* __restrict__ grad,
                                             const float* __restrict__ mem, float eta,
                                             double* __restrict__ partials, int32_t* done,
                                             int32_t* ready, float* __restrict__ scales,
                                             float* __restrict__ vals, int32_t* status,
                                             double* s_red, int* s_last) {
    const int tid = threadIdx.x;
    double acc = 0.0;
    if ((x.base & 3) == 0 && x.cnt == kTkTile) {
        const uint64_t pol = kKeep ? l2_evict_last_policy() : 0;
#pragma unroll
        for (int q = 0; q < kTkTile / 4 / 256; ++q) {
            const int e = 4 * (q * 256 + tid);
            const float4 g = kKeep ? ld_hint4(grad + x.base + e, pol)
                                   : ld_stream4(grad + x.base + e);
            const float4 m = kKeep ? ld_hint4(mem + x.base + e, pol)
                                   : *reinterpret_cast<const float4*>(mem + x.base + e);
            acc += fabs(double(residual(m.x, eta, g.x))) + fabs(double(residual(m.y, eta, g.y))) +
                   fabs(double(residual(m.z, eta, g.z))) + fabs(double(residual(m.w, eta, g.w)));
        }
    } else {
        for (int e = tid; e < x.cnt; e += 256)
            acc += fabs(double(residual(mem[x.base + e], eta, grad[x.base + e])));
    }
    // a NaN or infinite p makes the sum non-finite
    flag_nonfinite(!(fabs(acc) < 1.0e308), status);
    acc = block_sum_fixed(acc, s_red);
    if (tid == 0) {
        partials[t] = acc;
        __threadfence();
        *s_last = atomicAdd(&done[x.seg], 1) == x.L.ntiles - 1;
    }
    __syncthreads();
    if (*s_last) {  // the whole block adds the layer's partials (fixed order)
        __threadfence();
        const double* pp = partials + int64_t(x.w) * tiles_pw + x.L.tile0;
        double part = 0.0;
        for (int i = tid; i < x.L.ntiles; i += blockDim.x) part += __ldcg(pp + i);
        const double sum = block_sum_fixed(part, s_red);
        if (tid == 0) {
            const float s = float(sum / double(x.L.n));
            scales[x.seg] = s;
            float* slot = vals + int64_t(x.w) * vals_pw + x.L.val_off;
            slot[0] = s;
            slot[1] = slot[2] = slot[3] = 0.0f;
            if (ready) {
                __threadfence();
                st_release_gpu(ready + x.seg, 1);
            }
        }
    }
    __syncthreads();
}

// ---- emit of one tile: memory update and sign words ----------------------------------
__device__ __forceinline__ float sg_update(float p, float s, uint32_t& neg) {
    neg = __float_as_uint(p) >> 31;
    return neg ? __fadd_rn(p, s) : __fsub_rn(p, s);
}

// First sign word of the tile at element s0 of a layer whose payload starts
// at slot val_off (the scale and three pad slots come first).
__device__ __forceinline__ uint32_t* sg_words(float* vals, int64_t vals_pw, int w, int64_t val_off,
                                              int64_t s0) {
    return reinterpret_cast<uint32_t*>(vals + int64_t(w) * vals_pw + val_off + 4) + s0 / 32;
}

// words: the tile's first sign word; base: its first element in grad / mem.
// kHint: the second visit of the pipelined kernel, whose loads mark the lines
// evict-first (their last use).
template <bool kHint>
__device__ __forceinline__ void sg_emit_tile(int64_t base, int cnt, uint32_t* words, float s,
                                             const float* __restrict__ grad,
                                             float* __restrict__ mem, float eta) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e0 = warp * (kTkTile / 8);  // this warp's 1024 elements
    if ((base & 3) == 0 && cnt == kTkTile) {
        // all loads of the warp's 1024 elements first, then the updates
        float4 g[8], m[8];
        const uint64_t pol = kHint ? l2_evict_first_policy() : 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int e = e0 + 128 * q + 4 * lane;
            g[q] = kHint ? ld_hint4(grad + base + e, pol) : ld_stream4(grad + base + e);
            m[q] = kHint ? ld_hint4(mem + base + e, pol)
                         : *reinterpret_cast<const float4*>(mem + base + e);
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
            if (e < cnt)
                mem[base + e] = sg_update(residual(mem[base + e], eta, grad[base + e]), s, neg);
            const uint32_t word = __ballot_sync(kFull, neg != 0);
            if (lane == 0 && e0 + 32 * q < cnt) words[(e0 + 32 * q) / 32] = word;
        }
    }
}

// ---- two passes -----------------------------------------------------------------------
__global__ void __launch_bounds__(256) sg_norm_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t W, int32_t ncomp, int64_t N, int64_t vals_pw, const float* __restrict__ grad,
    const float* __restrict__ mem, float eta, double* __restrict__ partials,
    int32_t* __restrict__ done, float* __restrict__ scales, float* __restrict__ vals,
    int32_t* __restrict__ status) {
    grid_dependency_sync();
    __shared__ double s_red[8];
    __shared__ int s_last;
    for (int64_t t = blockIdx.x; t < int64_t(tiles_pw) * W; t += gridDim.x) {
        const SgTile x = sg_tile(layers, tile_layer, tiles_pw, ncomp, N, t);
        sg_norm_tile<false>(x, t, tiles_pw, vals_pw, grad, mem, eta, partials, done, nullptr,
                            scales, vals, status, s_red, &s_last);
    }
}

__global__ void __launch_bounds__(256) sg_emit_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t W, int32_t ncomp, int64_t N, int64_t vals_pw, const float* __restrict__ grad,
    float* __restrict__ mem, float eta, const float* __restrict__ scales,
    float* __restrict__ vals) {
    grid_dependency_sync();
    for (int64_t t = blockIdx.x; t < int64_t(tiles_pw) * W; t += gridDim.x) {
        const int w = int(t / tiles_pw);
        const int lt = int(t % tiles_pw);
        const DevLayer L = layers[tile_layer[lt]];
        const int64_t s0 = int64_t(lt - L.tile0) * kTkTile;
        sg_emit_tile<false>(int64_t(w) * N + L.offset + s0, int(min64(kTkTile, L.n - s0)),
                     sg_words(vals, vals_pw, w, L.val_off, s0), scales[int64_t(w) * ncomp + L.sidx],
                     grad, mem, eta);
    }
}

// ---- pipelined: one launch, norm tiles ahead of emit tiles -----------------------------
//
// Blocks take work items from a counter in a fixed order built on the host
// (sg_schedule): runs of norm tiles interleaved with runs of emit tiles, the
// norm tiles at most `ahead` tiles in front of the emit tiles, and every
// emit tile after all norm tiles of its layer.  An emit tile waits for its
// layer's scale.  Every item it can wait on was taken earlier by a running
// block (items go only to running blocks) that waits on nothing, so the wait
// ends; past kSgSpinLimit polls it sets GCE_STATUS_WAIT_TIMEOUT and carries
// on with whatever scale is there.
struct SgPhase {
    int64_t item0;  // first item of this run
    int64_t t0;     // its lowest tile
    int32_t kind;   // 0 norm, 1 emit, -1 end
    int32_t rev;    // 1: the run's tiles in descending order (item0 takes the highest)
};

constexpr uint32_t kSgSpinLimit = 1u << 21;  // polls (a sleep and an L2 load each): ~1 s

__global__ void __launch_bounds__(256, 4) sg_fused_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ tile_layer, int32_t tiles_pw,
    int32_t ncomp, int64_t N, int64_t vals_pw, const float* __restrict__ grad,
    float* __restrict__ mem, float eta, const SgPhase* __restrict__ phases, int32_t nphase,
    int64_t nitems, uint32_t* counter, double* __restrict__ partials, int32_t* done,
    int32_t* ready, float* __restrict__ scales, float* __restrict__ vals,
    int32_t* __restrict__ status) {
    grid_dependency_sync();
    __shared__ double s_red[8];
    __shared__ int s_last;
    __shared__ int64_t s_item;
    __shared__ int32_t s_ph;
    __shared__ float s_scale;
    const int tid = threadIdx.x;
    int ph = 0;  // thread 0's run: a block's items only increase
    for (;;) {
        if (tid == 0) {
            const int64_t it = int64_t(atomicAdd(counter, 1u));
            while (ph + 1 < nphase && phases[ph + 1].item0 <= it) ++ph;
            s_item = it;
            s_ph = ph;
        }
        __syncthreads();
        const int64_t it = s_item;
        if (it >= nitems) break;
        const SgPhase P = phases[s_ph];
        const int64_t off = it - P.item0;
        const int64_t t = P.rev ? P.t0 + (phases[s_ph + 1].item0 - P.item0 - 1 - off) : P.t0 + off;
        const SgTile x = sg_tile(layers, tile_layer, tiles_pw, ncomp, N, t);
        if (P.kind == 0) {
            sg_norm_tile<true>(x, t, tiles_pw, vals_pw, grad, mem, eta, partials, done, ready,
                               scales, vals, status, s_red, &s_last);
        } else {
            if (tid == 0) {
                int32_t r = ld_acquire_gpu(ready + x.seg);
                for (uint32_t n = 0; r == 0 && n < kSgSpinLimit; ++n) {
                    __nanosleep(128);
                    r = ld_acquire_gpu(ready + x.seg);
                }
                if (r == 0) atomicOr(status, GCE_STATUS_WAIT_TIMEOUT);
                s_scale = __ldcg(scales + x.seg);
            }
            __syncthreads();
            sg_emit_tile<true>(x.base, x.cnt, sg_words(vals, vals_pw, x.w, x.L.val_off, x.s0), s_scale,
                         grad, mem, eta);
        }
        __syncthreads();  // s_item, s_ph and s_scale are rewritten next
    }
}

// ---- majority vote ---------------------------------------------------------------------
// Majority vote of a SIGN table (SIGN and DENSE layers) for W <= 16 workers,
// one 4096-output tile per block step.  A warp takes the words of S worker
// slots (S the power of two at or above W) for 32 / S columns at a time: lane
// S c + w holds worker w's word c, and after a 32 x 32 bit transpose lane b
// holds bit b of every one of those words, the S-bit field c of which marks
// the workers with a negative sign at output 32 c + b; its population count is
// the vote.  A lane has kVoteBatch words in flight before their transposes,
// and every store writes 32 consecutive outputs.
constexpr int kVoteBatch = 8;

__global__ void __launch_bounds__(128) sg_vote_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ dc_tile_layer,
    int32_t dc_tiles, int32_t W, int64_t vals_pw, const float* __restrict__ vals, float scale,
    float* __restrict__ out) {
    grid_dependency_sync();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    int S = 1;
    while (S < W) S <<= 1;
    const int cols = 32 / S;                // columns a warp takes per transpose
    const int step = nwarps * cols;         // columns a block takes per transpose
    const int wk = lane & (S - 1), cl = lane / S;
    const uint32_t fmask = S == 32 ? 0xFFFFFFFFu : ((1u << S) - 1u);
    for (int32_t u = blockIdx.x; u < dc_tiles; u += gridDim.x) {
        const int32_t l = dc_tile_layer[u];
        const DevLayer L = layers[l];
        const int64_t start = int64_t(u - L.dc_tile0) << kDcTileLog;
        const int cnt = int(min64(kDcTile, L.n - start));
        float* o = out + L.offset + start;
        if (L.kind == GCE_KIND_SIGN) {
            const int nwords = (cnt + 31) >> 5;
            // worker wk's sign words of this tile (a lane with wk >= W reads none)
            const uint32_t* wp = reinterpret_cast<const uint32_t*>(
                                     vals + int64_t(wk < W ? wk : 0) * vals_pw + L.val_off + 4) +
                                 (start >> 5);
            for (int c0 = warp * cols; c0 < nwords; c0 += kVoteBatch * step) {
                uint32_t x[kVoteBatch];
#pragma unroll
                for (int b = 0; b < kVoteBatch; ++b) {
                    const int c = c0 + b * step + cl;
                    x[b] = (wk < W && c < nwords) ? __ldcg(wp + c) : 0u;
                }
#pragma unroll
                for (int b = 0; b < kVoteBatch; ++b) {
                    const int cb = c0 + b * step;  // the same for the whole warp
                    if (cb >= nwords) break;
                    const uint32_t neg = warp_transpose32(x[b]);
                    for (int cc = 0; cc < cols; ++cc) {
                        const int i = 32 * (cb + cc) + lane;
                        const int v = W - 2 * __popc((neg >> (S * cc)) & fmask);
                        if (i < cnt) o[i] = v > 0 ? scale : (v < 0 ? -scale : 0.0f);
                    }
                }
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

// The same vote for more than 16 workers: four outputs a thread, each worker's
// bits added one by one.  (With 32 worker slots a lane's word comes from its
// own worker, so every load of the transposed form touches 32 sectors; this
// form measured faster there.)
__global__ void __launch_bounds__(128) sg_vote_wide_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ dc_tile_layer,
    int32_t dc_tiles, int32_t W, int64_t vals_pw, const float* __restrict__ vals, float scale,
    float* __restrict__ out) {
    grid_dependency_sync();
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

// ---- host: the pipelined schedule, built once per (table, W, ahead) -------------------
constexpr int64_t kSgRun = 64;             // tiles per run of the schedule
constexpr int32_t kSgAuto = -1;            // look-ahead from the device's L2 size
constexpr int64_t kSgWaitTestTiles = 8;             // largest table (tiles) it runs on

// The order of the pipelined kernel's work items: runs of kSgRun norm tiles
// while the norm is fewer than `ahead` tiles in front, else a run of emit
// tiles, never past the first layer whose norm tiles are not all placed.
// ahead < 0 (the wait test): every emit run first, then every norm run.
// starts: the first tile of every (worker, layer), ascending; T tiles in all.
static std::vector<SgPhase> sg_schedule_of(const std::vector<int64_t>& starts, int64_t T,
                                           int32_t ahead, int64_t* nitems) {
    if (ahead < 0) {
        std::vector<SgPhase> ph;
        int64_t item = 0;
        for (int32_t kind = 1; kind >= 0; --kind)
            for (int64_t p = 0; p < T; p += kSgRun) {
                ph.push_back(SgPhase{item, p, kind, 0});
                item += std::min(T, p + kSgRun) - p;
            }
        ph.push_back(SgPhase{item, T, -1, 0});
        *nitems = item;
        return ph;
    }
    std::vector<SgPhase> ph;
    int64_t np = 0, ep = 0, item = 0;  // next norm tile, next emit tile
    // [first, end) tiles of the (worker, layer) holding tile x
    auto seg_of = [&](int64_t x, int64_t* first, int64_t* end) {
        const auto it = std::upper_bound(starts.begin(), starts.end(), x);
        *first = it == starts.begin() ? 0 : *(it - 1);
        *end = it == starts.end() ? T : *it;
    };
    while (ep < T) {
        // tiles below `limit` belong to layers whose norm tiles are all placed
        int64_t limit = T;
        if (np < T) {
            const auto it = std::upper_bound(starts.begin(), starts.end(), np);
            limit = it == starts.begin() ? 0 : *(it - 1);
        }
        const bool can_emit = limit > ep;
        if (np < T && (np - ep < ahead || !can_emit)) {
            const int64_t e = std::min(T, np + kSgRun);
            ph.push_back(SgPhase{item, np, 0, 0});
            item += e - np;
            np = e;
        } else {
            // A layer longer than the look-ahead is updated from its last tile
            // down: by the time its norm is complete only its last tiles are
            // still in L2, and they are read first.  Runs stop at the edges of
            // such a layer.
            int64_t first = 0, end = 0;
            seg_of(ep, &first, &end);
            const bool big = end - first > ahead;
            int64_t e = std::min(limit, ep + kSgRun);
            if (big) {
                e = std::min(e, end);
            } else {
                // stop before the first reversed layer inside the run
                for (int64_t x = end; x < e;) {
                    int64_t f2 = 0, e2 = 0;
                    seg_of(x, &f2, &e2);
                    if (e2 - f2 > ahead) {
                        e = x;
                        break;
                    }
                    x = e2;
                }
            }
            if (big)  // the mirror of [ep, e) inside [first, end)
                ph.push_back(SgPhase{item, first + end - e, 1, 1});
            else
                ph.push_back(SgPhase{item, ep, 1, 0});
            item += e - ep;
            ep = e;
        }
    }
    ph.push_back(SgPhase{item, T, -1, 0});
    *nitems = item;
    return ph;
}

static std::vector<SgPhase> sg_schedule(const gce_table* t, int32_t W, int32_t ahead,
                                        int64_t* nitems) {
    std::vector<int64_t> starts;
    starts.reserve(size_t(W) * t->comp.size());
    for (int32_t w = 0; w < W; ++w)
        for (int32_t l : t->comp) starts.push_back(int64_t(w) * t->tiles_pw + t->layers[l].tile0);
    std::sort(starts.begin(), starts.end());
    return sg_schedule_of(starts, int64_t(W) * t->tiles_pw, ahead, nitems);
}

// The look-ahead in tiles: the setting, or by default the tiles (grad and
// memory, 64 KB each) in 3/8 of the device's L2, rounded to whole runs.  The
// live window is about twice the look-ahead (norm tiles waiting for their
// update, plus the tiles in flight), which must stay in L2: on B200 (126 MB)
// this is 768 tiles, the best of the look-aheads measured there.
static int32_t sign_ahead_now(const gce_table* t) {
    const int32_t a = int32_t(option_of(t, GCE_OPT_SIGN_AHEAD));
    if (a != kSgAuto) return a;
    int dev = 0, l2 = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0) {
        cudaGetLastError();
        return 768;
    }
    const double tiles = double(l2) * 3.0 / 8.0 / double(kTkTile * 8);
    const int64_t r = std::llround(tiles / double(kSgRun)) * kSgRun;
    return int32_t(std::min<int64_t>(std::max<int64_t>(r, kSgRun), int64_t(1) << 20));
}

// The cached schedule of (W, ahead), built and uploaded on first use.  None
// while the stream is being captured (no synchronous copy then), or if the
// item counter could overflow: the caller then runs the two passes.
static bool sg_plan(const gce_table* t, int32_t W, int32_t ahead, cudaStream_t st, SgPlan* out) {
    std::lock_guard<std::mutex> lk(t->sg_mu);
    for (const SgPlan& p : t->sg_plans)
        if (p.W == W && p.ahead == ahead) {
            *out = p;
            return true;
        }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
        cudaGetLastError();
        return false;
    }
    int64_t nitems = 0;
    const std::vector<SgPhase> ph = sg_schedule(t, W, ahead, &nitems);
    if (nitems + (int64_t(1) << 24) >= (int64_t(1) << 32)) return false;
    void* d = nullptr;
    const size_t bytes = ph.size() * sizeof(SgPhase);
    if (cudaMalloc(&d, bytes) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (cudaMemcpy(d, ph.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(d);
        return false;
    }
    const SgPlan p{W, ahead, int32_t(ph.size()), nitems, d};
    t->sg_plans.push_back(p);
    *out = p;
    return true;
}

void sign_plan_free(gce_table* t) {
    for (const SgPlan& p : t->sg_plans) cudaFree(p.d_phases);
    t->sg_plans.clear();
}

}  // namespace gce

using namespace gce;

extern "C" int gce_sign_schedule(const int32_t* layer_tiles, int32_t ncomp, int32_t W,
                                 int32_t ahead, int64_t* runs, int64_t cap, int64_t* nruns) {
    if (!layer_tiles || ncomp < 1 || W < 1 || ahead < -1 || ahead > (1 << 20) || !nruns ||
        cap < 0 || (cap > 0 && !runs))
        return GCE_ERR_ARG;
    int64_t tiles_pw = 0;
    std::vector<int64_t> tile0(size_t(ncomp), 0);
    for (int32_t l = 0; l < ncomp; ++l) {
        if (layer_tiles[l] < 1) return GCE_ERR_ARG;
        tile0[l] = tiles_pw;
        tiles_pw += layer_tiles[l];
    }
    std::vector<int64_t> starts;
    starts.reserve(size_t(W) * size_t(ncomp));
    for (int32_t w = 0; w < W; ++w)
        for (int32_t l = 0; l < ncomp; ++l) starts.push_back(int64_t(w) * tiles_pw + tile0[l]);
    int64_t nitems = 0;
    const std::vector<SgPhase> ph = sg_schedule_of(starts, int64_t(W) * tiles_pw, ahead, &nitems);
    *nruns = int64_t(ph.size());
    for (int64_t i = 0; i < std::min<int64_t>(cap, int64_t(ph.size())); ++i) {
        runs[4 * i] = ph[size_t(i)].item0;
        runs[4 * i + 1] = ph[size_t(i)].t0;
        runs[4 * i + 2] = ph[size_t(i)].kind;
        runs[4 * i + 3] = ph[size_t(i)].rev;
    }
    return GCE_OK;
}

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
        const int64_t segs = int64_t(W) * ncomp;
        const int64_t tiles = int64_t(t->tiles_pw) * W;
        const bool emit_first = option_of(t, GCE_OPT_SIGN_EMIT_FIRST) != 0.0;
        // the wait test: every update's wait runs out, one block after another,
        // so it is refused beyond a few tiles
        if (emit_first && tiles > kSgWaitTestTiles) return GCE_ERR_ARG;
        int32_t* done = at<int32_t>(ws, lay.sync);
        int32_t* ready = done + segs;
        uint32_t* counter = reinterpret_cast<uint32_t*>(done + 2 * segs);
        if (cudaMemsetAsync(done, 0, sizeof(int32_t) * size_t(2 * segs + 1), st) != cudaSuccess)
            return GCE_ERR_CUDA;
        const int32_t ahead = emit_first ? -1 : sign_ahead_now(t);
        SgPlan plan;
        if (ahead != 0 && sg_plan(t, W, ahead, st, &plan)) {
            static const int r_fused = resident_blocks(sg_fused_kernel, 256);
            // the wait test runs one block, so no norm tile runs while it waits
            const int grid = ahead < 0 ? 1 : wave_grid(plan.nitems, 8, r_fused);
            GCE_LAUNCH(sg_fused_kernel, grid, 256, 0, st,
                       t->d_layers, t->d_tile_layer, t->tiles_pw, ncomp, t->N, t->vals_pw, grad,
                       mem, eta, static_cast<const SgPhase*>(plan.d_phases), plan.nphase,
                       plan.nitems, counter, at<double>(ws, lay.partials), done, ready,
                       at<float>(ws, lay.scales), vals, status);
        } else {
            static const int r_norm = resident_blocks(sg_norm_kernel, 256);
            static const int r_emit = resident_blocks(sg_emit_kernel, 256);
            GCE_LAUNCH(sg_norm_kernel, wave_grid(tiles, 8, r_norm), 256, 0, st, t->d_layers,
                       t->d_tile_layer, t->tiles_pw, W, ncomp, t->N, t->vals_pw, grad, mem, eta,
                       at<double>(ws, lay.partials), done, at<float>(ws, lay.scales), vals,
                       status);
            GCE_LAUNCH(sg_emit_kernel, wave_grid(tiles, 8, r_emit), 256, 0, st, t->d_layers,
                       t->d_tile_layer, t->tiles_pw, W, ncomp, t->N, t->vals_pw, grad, mem, eta,
                       at<float>(ws, lay.scales), vals);
        }
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
    static const int r_vote_wide = resident_blocks(sg_vote_wide_kernel, 128);
    if (t->dc_tiles > 0 && W <= 16)
        GCE_LAUNCH(sg_vote_kernel, wave_grid(t->dc_tiles, 16, r_vote), 128, 0, st, t->d_layers,
                   t->d_dc_tile_layer, t->dc_tiles, W, t->vals_pw, vals, scale, out);
    else if (t->dc_tiles > 0)
        GCE_LAUNCH(sg_vote_wide_kernel, wave_grid(t->dc_tiles, 16, r_vote_wide), 128, 0, st,
                   t->d_layers, t->d_dc_tile_layer, t->dc_tiles, W, t->vals_pw, vals, scale, out);
    return check_launch();
}
