// common.cuh -- shared internals of the gce library (sm_100a): the layer
// table, workspace carving, launch accounting and small device helpers.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <utility>
#include <cstddef>
#include <cstdint>
#include <mutex>
#include <vector>

#include "gce.h"

namespace gce {

constexpr int kMaxRank = 4;

// Device copy of one layer.  Offsets are in elements (grad/mem), slots
// (vals/idx) or floats (P, Q) per worker.
struct DevLayer {
    int64_t offset, n, rows, cols;
    int64_t val_off, p_off, q_off;
    int64_t sp_off;  // offset among the compressed layers' elements (spill slots)
    int32_t kind, cap;
    int32_t tile0, ntiles;  // top-k / rand-k main tiles of this layer, per worker
    int32_t sidx;           // index among compressed layers, -1 for DENSE
    int32_t dc_tile0;       // first decode tile of this layer (all layers, per table)
    int32_t dc_ntiles;      // decode tiles of this layer
    int32_t dc_base;        // first slot of this layer's nspans+1 span bounds
};

// One main tile's layer fields, for kernels whose per-tile work is short:
// one 32-byte load instead of tile -> layer id -> layer record.
struct alignas(16) TileInfo {
    int64_t offset;   // first element of the tile's layer in a worker's buffer
    int64_t sp_off;   // the layer's first candidate slot
    int64_t val_off;  // the layer's first payload slot
    int32_t sidx;     // index among the compressed layers
    int32_t tstart;   // first element of the tile within its layer
};

// One TOPK / RANDK decode tile's fields, stored in the order the sparse decoder
// takes the tiles: its per-span work starts from one 48-byte record instead of
// tile -> layer id -> layer record.
struct alignas(16) DcTileInfo {
    int64_t out_off;  // first output of the tile (layer offset + tstart)
    int64_t val_off;  // the layer's first payload slot
    int32_t tstart;   // first element of the tile within its layer
    int32_t cnt;      // outputs in the tile: kDcTile, or fewer at the layer's end
    int32_t bslot;    // span-bound slot of the tile's first span
    int32_t layer;    // layer id, for a per-layer k
    int32_t cap;      // the layer's cap on k
    int32_t pad[3];
};

// A pipelined signSGD schedule uploaded for one (W, ahead): nphase runs
// (the last a sentinel) covering nitems work items.
struct SgPlan {
    int32_t W, ahead, nphase;
    int64_t nitems;
    void* d_phases;
};

}  // namespace gce

struct gce_table {
    int32_t L = 0;
    int64_t N = 0, vals_pw = 0, P_pw = 0, Q_pw = 0;
    int32_t ckind = -1;
    std::vector<gce::DevLayer> layers;     // host copy
    gce::DevLayer* d_layers = nullptr;
    std::vector<int32_t> comp;             // compressed layer ids, in order
    std::vector<int32_t> dense;            // DENSE layer ids
    int32_t* d_comp = nullptr;
    int32_t* d_dense = nullptr;
    int64_t comp_N = 0;                    // elements in compressed layers, per worker
    int64_t dense_N = 0;
    int64_t max_comp_n = 0;
    int32_t tiles_pw = 0;                  // main tiles (compressed layers) per worker
    int32_t* d_tile_layer = nullptr;       // [tiles_pw] layer of each main tile
    gce::TileInfo* d_tile_info = nullptr;  // [tiles_pw] the same tiles' layer fields
    int32_t sunits_pw = 0;                 // top-k sample units per worker
    int32_t* d_sunit_layer = nullptr;      // [sunits_pw] layer of each sample unit
    int32_t* d_sunit_part = nullptr;       // [sunits_pw] part index within the layer
    int32_t dtiles_pw = 0;                 // dense-layer tiles per worker
    int32_t* d_dtile_layer = nullptr;
    int32_t* d_dtile_start = nullptr;      // element start of each dense tile
    int32_t dc_tiles = 0;                  // decode tiles over all layers
    int32_t dc_slots = 0;                  // span-bound slots per worker (spans + L)
    int32_t* d_dc_tile_layer = nullptr;    // [dc_tiles] layer of each decode tile
    int32_t dc_nl_n = 0;                   // decode tiles of sparse and DENSE layers
    int32_t* d_dc_nl_tiles = nullptr;      // their decode tile ids
    int32_t dc_sp_n = 0;                   // decode tiles of TOPK and RANDK layers
    gce::DcTileInfo* d_dc_sp_info = nullptr;  // their fields, in decode order
    int32_t dc_dn_n = 0;                   // decode tiles of DENSE layers
    int32_t* d_dc_dn_tiles = nullptr;      // their decode tile ids
    int32_t bunits_pw = 0;                 // decode bound units (sparse layers) per worker
    int32_t* d_bunit_layer = nullptr;
    int32_t* d_bunit_chunk = nullptr;
    // PowerSGD plan (built by gce::powersgd_plan)
    void* d_ps = nullptr;                  // PsLayer[L]
    int4* d_ps1_tiles = nullptr;           // (layer, row block, column chunk) of M Q and residual
    int32_t ps1_ntiles = 0;
    int32_t ps1_nexact = 0;                // the first ps1_nexact of them: fp64-product layers
    int4* d_ps3_tiles = nullptr;           // (layer, row block, column chunk) of M^T P
    int32_t ps3_ntiles = 0;
    int32_t ps3_nexact = 0;
    int4* d_psq_tiles = nullptr;           // (layer, column block) of the Q reduction
    int32_t psq_ntiles = 0;
    int32_t* d_ps_layers = nullptr;        // POWERSGD layer ids
    int32_t nps = 0;
    int64_t ppart_pw = 0, pd_pw = 0, qpart_pw = 0;  // workspace floats / doubles per worker
    int32_t ps_ntall = 0, ps_tall_parts = 0, ps_tall_cap = 0, ps_tall_nunits = 0;
    int2* d_ps_tall_units = nullptr;       // (layer, row chunk) of tall P matrices
    // Accordion plan (built by gce::accordion_plan)
    int2* d_ac_tiles = nullptr;            // (layer, chunk) of the norm reduction
    int32_t ac_ntiles = 0;
    int2* d_ac_layer = nullptr;            // per layer: (first norm tile, tile count)
    // rand-k: the key pass the last ef_randk_step ran ahead for the next step
    // (step rk_step, seed rk_seed, W rk_W workers from rk_worker0) in workspace
    // rk_ws; guarded by rk_mu
    mutable std::mutex rk_mu;
    mutable const void* rk_ws = nullptr;
    mutable uint64_t rk_seed = 0, rk_step = 0;
    mutable int32_t rk_W = 0;
    mutable int64_t rk_worker0 = 0;
    mutable bool rk_valid = false;
    // signSGD: pipelined schedules by (W, ahead), kept until the table is
    // destroyed; guarded by sg_mu
    mutable std::mutex sg_mu;
    mutable std::vector<gce::SgPlan> sg_plans;
    // settings of this table (gce_table_set_option), one per GCE_OPT_*; NaN:
    // follow the process-wide setting
    std::atomic<double> opt[4] = {NAN, NAN, NAN, NAN};
};

namespace gce {

// ---- launch accounting -------------------------------------------------
extern std::atomic<uint64_t> g_launches;

inline void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// optional per-launch timing: two events on the launch's stream around it
extern std::atomic<bool> g_prof_on;
void prof_before(const char* name, cudaStream_t st);
void prof_after(cudaStream_t st);

// Every kernel of the library is launched with programmatic stream
// serialisation allowed: its blocks may be scheduled while the kernel before
// it in the stream drains, and each kernel's first statement,
// grid_dependency_sync(), holds them until that kernel has completed and its
// writes are visible.  The setting is read once from the environment
// (GCE_PROGRAMMATIC_LAUNCH=0 turns it off); results do not depend on it.
bool programmatic_launch();

template <class... KArgs, class... Args>
inline void launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, Args&&... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic_launch() ? 1 : 0;
    // a failed launch is reported by the caller's check_launch()
    (void)cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

#define GCE_LAUNCH(kern, grid, block, smem, stream, ...)                        \
    do {                                                                         \
        ::gce::count_launch();                                                   \
        const bool gce_prof_ = ::gce::g_prof_on.load(std::memory_order_relaxed); \
        if (gce_prof_) ::gce::prof_before(#kern, (stream));                      \
        ::gce::launch_kernel(kern, (grid), (block), (smem), (stream), __VA_ARGS__); \
        if (gce_prof_) ::gce::prof_after((stream));                              \
    } while (0)

// The same with the name recorded for the profile given as a string, for a
// kernel whose template arguments hold a comma (written with GCE_COMMA).
#define GCE_COMMA ,
#define GCE_LAUNCH_AS(name, kern, grid, block, smem, stream, ...)               \
    do {                                                                         \
        ::gce::count_launch();                                                   \
        const bool gce_prof_ = ::gce::g_prof_on.load(std::memory_order_relaxed); \
        if (gce_prof_) ::gce::prof_before((name), (stream));                     \
        ::gce::launch_kernel(kern, (grid), (block), (smem), (stream), __VA_ARGS__); \
        if (gce_prof_) ::gce::prof_after((stream));                              \
    } while (0)

// First statement of every kernel: wait until the kernel this launch depends
// on in its stream has completed and its writes are visible (immediate when
// the launch was not programmatic), then let the next launch in the stream
// be scheduled.  Blocks of that launch wait in their own first statement, so
// no kernel reads or writes memory while its predecessor still runs.
__device__ __forceinline__ void grid_dependency_sync() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

inline int check_launch() {
    return cudaGetLastError() == cudaSuccess ? GCE_OK : GCE_ERR_CUDA;
}

// ---- settings that move work or test a wait ------------------------------------
// The value a call on table t uses for option `opt` (GCE_OPT_*): the table's
// own, else the process-wide one.  Read once per call.
double option_of(const gce_table* t, int opt);

// ---- device properties (cached per device) --------------------------------
int sm_count();

// ---- grids -------------------------------------------------------------------
// Blocks of `kernel` (`threads` threads, no dynamic shared memory) that fit on
// one SM at once.
template <class K>
inline int resident_blocks(K kernel, int threads) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1)
        n = 1;
    return n;
}

// The same for a kernel with `smem` bytes of dynamic shared memory; allows the
// kernel that much (above the 48 KB default) on the current device first.
template <class K>
inline int resident_blocks_smem(K kernel, int threads, size_t smem) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
        cudaGetLastError();
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess ||
        n < 1) {
        cudaGetLastError();
        n = 1;
    }
    return n;
}

// Grid of a grid-stride kernel: at most `per_sm` blocks per SM and never more
// than fit at once (`resident`), so the whole grid runs in one wave.  A block
// of a second, partial wave would start only when a first-wave block had
// finished all of its tiles, nearly doubling the kernel's time.
inline int wave_grid(int64_t work, int per_sm, int resident) {
    const int p = per_sm < resident ? per_sm : resident;
    const int64_t cap = int64_t(sm_count()) * p;
    return int(work < 1 ? 1 : (work < cap ? work : cap));
}

// (worker, tile within the worker) along a grid-stride walk over W x tiles_pw
// tiles: one division at the start, then each step adds the stride's whole
// workers and remaining tiles, carrying one worker when the tile overflows.
struct TileWalk {
    int64_t t;
    int32_t w, lt, dw, dlt, tiles_pw;
    __device__ __forceinline__ TileWalk(int64_t t0, int64_t stride, int32_t tpw)
        : t(t0), tiles_pw(tpw) {
        w = int32_t(t0 / tpw);
        lt = int32_t(t0 - int64_t(w) * tpw);
        dw = int32_t(stride / tpw);
        dlt = int32_t(stride - int64_t(dw) * tpw);
    }
    __device__ __forceinline__ void next(int64_t stride) {
        t += stride;
        w += dw;
        lt += dlt;
        if (lt >= tiles_pw) {
            lt -= tiles_pw;
            ++w;
        }
    }
};

// ---- workspace carving ------------------------------------------------------
struct Carver {
    size_t off = GCE_WS_HEADER_BYTES;
    template <class T>
    size_t take(size_t count) {
        size_t o = off;
        off += (count * sizeof(T) + 255) & ~size_t(255);
        return o;
    }
};

template <class T>
inline T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- device helpers -----------------------------------------------------------
__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

__device__ __forceinline__ void set_status(int32_t* status, int32_t bit) {
    atomicOr(status, bit);
}

// Mem-SGD residual v = fl32(m + fl32(eta*g)): explicit round-to-nearest
// multiply then add, never contracted into an FMA.
__device__ __forceinline__ float residual(float m, float eta, float g) {
    return __fadd_rn(m, __fmul_rn(eta, g));
}

// Last step of every decoder: out = fl(scale * s), or, fused with the
// parameter update x_{t+1} = x_t - g_t (kApply), x = fl(x - fl(scale * s)).
template <bool kApply>
__device__ __forceinline__ float dc_final(float s, float scale, const float* o) {
    const float u = __fmul_rn(s, scale);
    return kApply ? __fsub_rn(*o, u) : u;
}

template <bool kApply>
__device__ __forceinline__ float4 dc_final4(float4 s, float scale, const float4* o4) {
    float4 u = make_float4(__fmul_rn(s.x, scale), __fmul_rn(s.y, scale), __fmul_rn(s.z, scale),
                           __fmul_rn(s.w, scale));
    if (kApply) {
        const float4 x = __ldcs(o4);
        u = make_float4(__fsub_rn(x.x, u.x), __fsub_rn(x.y, u.y), __fsub_rn(x.z, u.z),
                        __fsub_rn(x.w, u.w));
    }
    return u;
}

// Keys at or above this one (sign cleared) belong to +-Inf and NaN.
constexpr uint32_t kNonFiniteKey = 0x7F800000u;

// Sets GCE_STATUS_NONFINITE if any lane saw a non-finite value.  Call with
// the whole warp.
__device__ __forceinline__ void flag_nonfinite(bool bad, int32_t* status) {
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0)
        atomicOr(status, GCE_STATUS_NONFINITE);
}

// |v| ordering key: the float's bits with the sign cleared.
__device__ __forceinline__ uint32_t abs_key(float v) {
    return __float_as_uint(v) & 0x7FFFFFFFu;
}

__device__ __forceinline__ float4 ld_stream4(const float* p) {
    return __ldcs(reinterpret_cast<const float4*>(p));
}

// Acquire / release accesses at GPU scope, for flags that one block publishes
// and blocks of the same launch wait on.
__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t* p) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(int32_t* p, int32_t v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint64_t ld_acquire_gpu_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.release.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Bulk (TMA-engine) prefetch of a contiguous range into L2: one instruction
// for `bytes` (a multiple of 16) starting at a 16-byte aligned address.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// host entry points shared between translation units
constexpr int kDcTileLog = 12;              // decode tile: 4096 output elements
constexpr int kDcTile = 1 << kDcTileLog;
constexpr int kDcSpanLog = 10;              // decode span: 1024 outputs, a warp's share
constexpr int kDcSpan = 1 << kDcSpanLog;    // of a tile; payload entry bounds per span
constexpr int kDcBoundChunk = 8192;         // payload entries per bound unit
constexpr int kDenseTile = 4096;            // elements per tile of a DENSE layer

void sign_plan_free(gce_table* t);
int launch_dense_layers(const gce_table* t, int32_t W, const float* grad, float* mem,
                        float eta, float* vals, int32_t* status, cudaStream_t st);
bool launch_lowrank_decode(const gce_table* t, int32_t W, const int32_t* k_or_rank,
                           const float* P, const float* Q, float scale, float* out, bool apply,
                           cudaStream_t st);
int powersgd_plan(gce_table* t);   // called once by gce_table_create
void powersgd_plan_free(gce_table* t);
int accordion_plan(gce_table* t);  // called once by gce_table_create
void accordion_plan_free(gce_table* t);

// SplitMix64 (Steele, Lea, Flood 2014): 64-bit finaliser and golden gamma
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// The high 32 bits of mix64(z), forming only the high word of the last
// product (the same value: the final xor-shift moves bit 63 into bit 32
// and leaves the high word otherwise as it is).
__host__ __device__ __forceinline__ uint32_t mix64_hi(uint64_t z) {
    const uint64_t y0 = z ^ (z >> 30);
    const uint64_t z1 = y0 * 0xBF58476D1CE4E5B9ull;
    const uint64_t y1 = z1 ^ (z1 >> 27);
    const uint32_t lo = uint32_t(y1), hi = uint32_t(y1 >> 32);
    constexpr uint32_t c_lo = 0x133111EBu, c_hi = 0x94D049BBu;
#ifdef __CUDA_ARCH__
    const uint32_t h = __umulhi(lo, c_lo) + lo * c_hi + hi * c_lo;
#else
    const uint32_t h = uint32_t((uint64_t(lo) * c_lo) >> 32) + lo * c_hi + hi * c_lo;
#endif
    return h ^ (h >> 31);
}

// state of (seed, stream, worker, layer, step): each field folded in as the
// first SplitMix64 output from (previous + (field + 1) * gamma)
__host__ __device__ __forceinline__ uint64_t hash_base(uint64_t seed, uint64_t stream,
                                                       uint64_t worker, uint64_t layer,
                                                       uint64_t step) {
    uint64_t h = mix64(seed + (stream + 1) * kGamma);
    h = mix64(h + (worker + 1) * kGamma);
    h = mix64(h + (layer + 1) * kGamma);
    h = mix64(h + (step + 1) * kGamma);
    return h;
}

}  // namespace gce
