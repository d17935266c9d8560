// powersgd.cu -- PowerSGD rank-r compression with error feedback on sm_100a.
//
// The pages name PowerSGD and its ranks ("Accordion ...", Method and Key
// results: ranks 1/2/4; "On the Utility of Gradient Compression ...", Method
// and Key results: all-reduce compatible) without printing its steps; this
// file implements the standard single power-iteration step with a reused Q,
// with the Mem-SGD memory of "Sparsified SGD with Memory", Method:
//   M = fl(m + fl(eta*g))                         (residual, as Mem-SGD)
//   P = M Q            (Q: warm start, cols x r)
//   P <- orthonormal columns (modified Gram-Schmidt, column order, fp64)
//   Q <- M^T P
//   m <- M - P Q^T,  dense_out <- P Q^T
//
// r <= 4, so every product is a skinny contraction of about 2r flops per
// element of M: far below the tensor-core ridge and below the CUDA-core one,
// so the kernels are plain register-blocked FMA loops shaped for bandwidth:
//   mq      one pass over grad and mem: M written back to mem, and per
//           (row block, 1024-column chunk) tile each warp reduces its rows
//           against the Q chunk staged in shared memory -> partial P; row
//           blocks of 64 rows in layers of at least 2^24 elements, 16 below
//   orth    one CTA per matrix: partial P summed in fp64 in chunk order,
//           then Gram-Schmidt with fp64 block reductions in a fixed order
//   mtp     per (row block, 1024-column chunk): each thread owns 4
//           columns and accumulates M^T P over the block's rows -> partials;
//           256-row blocks in layers of at least 2^24 elements, 64 below
//   qred    the row-block partials summed in fp64 in block order -> Q
//   resid   m <- M - P Q^T with the same product order as the decoder
// DRAM traffic for matrices that stay in L2 between the passes: 12 B per
// element (read grad, read mem, write mem once); otherwise mtp and resid
// re-read M (+8 B) and resid writes it (+4 B; +4 B for dense_out).
#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "scan.cuh"

namespace gce {

constexpr int kPsRB = 64;     // most rows per M Q / residual / decode tile
constexpr int kPsRBSmall = 16;                     // rows per such tile of a layer
constexpr int64_t kPsTallTileMin = int64_t(1) << 24;  // smaller than this many elements
constexpr int kPsCB = 1024;   // columns per chunk (256 threads x 4)
constexpr int kPsRB3 = 256;   // most rows per M^T P tile (its partial's row block)
constexpr int kPsRB3Small = 64;  // rows per such block of a layer under kPsTallTileMin elements
constexpr int kPsQB = 128;    // columns per Q-reduction tile
constexpr int kPsQBSplit = 32; // the same for a layer whose sums are split over four lanes
constexpr int kPsQSplit = 32; // row blocks from which four lanes share a Q entry's sum

constexpr int64_t kPsTallRows = 8192;  // taller P: Gram-Schmidt spread over many blocks
constexpr int kPsOrthChunk = 256;      // rows per block in that case

// Precision of a layer's products.  Layers of at most kPsExactMax elements
// form M Q, M^T P and the residual in fp64, from the fp64 orthonormal P and
// Q' (the oracle's arithmetic up to the order of fp64 sums); their tiles come
// first in the tile lists, and each precision has its own kernel instances.  B200's CUDA
// cores run fp64 at about 1/32 of the fp32 rate, which would make a larger,
// bandwidth-bound layer ALU-bound; larger layers form the products in fp32
// (per lane, from the fp32-rounded P and Q' the payload carries) and every
// sum across lanes, chunks and row blocks in fp64.
constexpr int64_t kPsExactMax = int64_t(1) << 22;

struct PsLayer {
    int64_t ppart_off;  // floats: nch1 x rows x cap partial P
    int64_t pd_off;     // doubles: rows x cap
    int64_t qpart_off;  // floats: nrb3 x cols x cap partial Q
    int32_t nch1, nrb3;
    int32_t tall;       // index among the tall layers, -1 otherwise
    int32_t part_off;   // first partial-sum slot of a tall layer
    int32_t nchunk;     // row chunks of a tall layer
    int32_t rb3;        // rows per M^T P block
};

int powersgd_plan(gce_table* t) {
    std::vector<PsLayer> ps(t->L);
    std::vector<int4> t1, t3, tq, t1f, t3f;
    std::vector<int2> tall_units;
    std::vector<int32_t> ids;
    int64_t pp = 0, pd = 0, qp = 0;
    int32_t ntall = 0, nparts = 0, tall_cap = 0;
    for (int32_t l = 0; l < t->L; ++l) {
        const DevLayer& L = t->layers[l];
        PsLayer x{};
        x.tall = -1;
        if (L.kind == GCE_KIND_POWERSGD && L.rows > kPsTallRows) {
            x.tall = ntall++;
            x.nchunk = int32_t((L.rows + kPsOrthChunk - 1) / kPsOrthChunk);
            x.part_off = nparts;
            nparts += x.nchunk;
            tall_cap = std::max(tall_cap, L.cap);
            for (int32_t c = 0; c < x.nchunk; ++c) tall_units.push_back(make_int2(l, c));
        }
        if (L.kind == GCE_KIND_POWERSGD) {
            x.nch1 = int32_t((L.cols + kPsCB - 1) / kPsCB);
            x.rb3 = L.n >= kPsTallTileMin ? kPsRB3 : kPsRB3Small;
            x.nrb3 = int32_t((L.rows + x.rb3 - 1) / x.rb3);
            x.ppart_off = pp;
            x.pd_off = pd;
            x.qpart_off = qp;
            pp += int64_t(x.nch1) * L.rows * L.cap;
            pd += L.rows * L.cap;
            qp += int64_t(x.nrb3) * L.cols * L.cap;
            // tiles of the fp64-product layers first, then the others
            const bool exact = L.n <= kPsExactMax;
            std::vector<int4>& o1 = exact ? t1 : t1f;
            std::vector<int4>& o3 = exact ? t3 : t3f;
            // (layer, first row, column chunk, rows): large layers in taller
            // tiles, which stage their factors once for more rows
            const int64_t rbh = L.n >= kPsTallTileMin ? kPsRB : kPsRBSmall;
            for (int64_t r0 = 0; r0 < L.rows; r0 += rbh)
                for (int32_t ch = 0; ch < x.nch1; ++ch)
                    o1.push_back(make_int4(l, int32_t(r0), ch, int32_t(std::min(rbh, L.rows - r0))));
            for (int32_t rb = 0; rb < x.nrb3; ++rb)
                for (int32_t ch = 0; ch < x.nch1; ++ch) o3.push_back(make_int4(l, rb, ch, 0));
            // Q-reduction tiles (layer, first column, columns): narrower where
            // four lanes share each entry's sum
            const int64_t qw = x.nrb3 >= kPsQSplit ? kPsQBSplit : kPsQB;
            for (int64_t c0 = 0; c0 < L.cols; c0 += qw)
                tq.push_back(make_int4(l, int32_t(c0), int32_t(std::min(qw, L.cols - c0)), 0));
            ids.push_back(l);
        }
        ps[l] = x;
    }
    t->ps1_nexact = int32_t(t1.size());
    t->ps3_nexact = int32_t(t3.size());
    t1.insert(t1.end(), t1f.begin(), t1f.end());
    t3.insert(t3.end(), t3f.begin(), t3f.end());
    t->ppart_pw = pp;
    t->pd_pw = pd;
    t->qpart_pw = qp;
    t->ps1_ntiles = int32_t(t1.size());
    t->ps3_ntiles = int32_t(t3.size());
    t->psq_ntiles = int32_t(tq.size());
    t->nps = int32_t(ids.size());
    t->ps_ntall = ntall;
    t->ps_tall_parts = nparts;
    t->ps_tall_cap = tall_cap;
    t->ps_tall_nunits = int32_t(tall_units.size());
    auto up = [](void** dst, const void* src, size_t bytes) -> int {
        *dst = nullptr;
        if (bytes == 0) return GCE_OK;
        if (cudaMalloc(dst, bytes) != cudaSuccess) return GCE_ERR_NOMEM;
        return cudaMemcpy(*dst, src, bytes, cudaMemcpyHostToDevice) == cudaSuccess ? GCE_OK
                                                                                  : GCE_ERR_CUDA;
    };
    int rc = up(&t->d_ps, ps.data(), ps.size() * sizeof(PsLayer));
    if (rc == GCE_OK) rc = up(reinterpret_cast<void**>(&t->d_ps1_tiles), t1.data(), t1.size() * sizeof(int4));
    if (rc == GCE_OK) rc = up(reinterpret_cast<void**>(&t->d_ps3_tiles), t3.data(), t3.size() * sizeof(int4));
    if (rc == GCE_OK) rc = up(reinterpret_cast<void**>(&t->d_psq_tiles), tq.data(), tq.size() * sizeof(int4));
    if (rc == GCE_OK) rc = up(reinterpret_cast<void**>(&t->d_ps_layers), ids.data(), ids.size() * sizeof(int32_t));
    if (rc == GCE_OK)
        rc = up(reinterpret_cast<void**>(&t->d_ps_tall_units), tall_units.data(),
                tall_units.size() * sizeof(int2));
    return rc;
}

void powersgd_plan_free(gce_table* t) {
    cudaFree(t->d_ps_tall_units);
    cudaFree(t->d_ps);
    cudaFree(t->d_ps1_tiles);
    cudaFree(t->d_ps3_tiles);
    cudaFree(t->d_psq_tiles);
    cudaFree(t->d_ps_layers);
}

struct PsWs {
    size_t ppart = 0, pd = 0, qpart = 0, qd = 0, qloc = 0, tparts = 0, tscal = 0, tdone = 0,
           total = 0;
};

// pd and qd hold the last step's fp64 orthonormal P and Q' (the lazy step
// takes its residual from them); the partial sums are fp64 too.
static PsWs ps_layout(const gce_table* t, int32_t W) {
    PsWs o;
    Carver c;
    o.ppart = c.take<double>(int64_t(W) * t->ppart_pw);
    o.pd = c.take<double>(int64_t(W) * t->pd_pw);
    o.qpart = c.take<double>(int64_t(W) * t->qpart_pw);
    o.qd = c.take<double>(int64_t(W) * t->Q_pw);
    o.tparts = c.take<double>(int64_t(W) * t->ps_tall_parts);
    o.tscal = c.take<double>(int64_t(W) * t->ps_ntall);
    o.tdone = c.take<int32_t>(int64_t(W) * t->ps_ntall);
    o.total = c.off;
    return o;
}

size_t powersgd_ws_bytes(const gce_table* t, int32_t W) { return ps_layout(t, W).total; }

// The data-parallel step: partials per worker, one orthonormal P per layer,
// and every worker's Q_w (fp32 for the mean, fp64 for its residual).
// The parts that do not grow with W come first, so that the orthonormalisation
// of a step split between ranks finds them at the same place whatever W the
// workspace was sized for.
static PsWs ps_dp_layout(const gce_table* t, int32_t W) {
    PsWs o;
    Carver c;
    o.pd = c.take<double>(t->pd_pw);
    o.tparts = c.take<double>(t->ps_tall_parts);
    o.tscal = c.take<double>(t->ps_ntall);
    o.tdone = c.take<int32_t>(t->ps_ntall);
    o.ppart = c.take<double>(int64_t(W) * t->ppart_pw);
    o.qpart = c.take<double>(int64_t(W) * t->qpart_pw);
    o.qd = c.take<double>(int64_t(W) * t->Q_pw);
    o.qloc = c.take<float>(int64_t(W) * t->Q_pw);
    o.total = c.off;
    return o;
}

size_t powersgd_dp_ws_bytes(const gce_table* t, int32_t W) { return ps_dp_layout(t, W).total; }

__device__ __forceinline__ int32_t ps_rank(const DevLayer& L, const int32_t* k_or_rank, int32_t l) {
    const int32_t r = k_or_rank ? k_or_rank[l] : L.cap;
    return (r >= 1 && r <= L.cap) ? r : 0;
}

// ---- Q initialisation --------------------------------------------------------------
__global__ void ps_init_q_kernel(const DevLayer* __restrict__ layers,
                                 const int32_t* __restrict__ ps_layers, int32_t nps, int32_t W,
                                 int64_t Q_pw, uint64_t seed, float* __restrict__ Q) {
    grid_dependency_sync();
    for (int64_t u = blockIdx.x; u < int64_t(nps) * W; u += gridDim.x) {
        const int w = int(u / nps);
        const int32_t l = ps_layers[u % nps];
        const DevLayer L = layers[l];
        const uint64_t base = hash_base(seed, 1, uint64_t(w), uint64_t(l), 0);
        float* q = Q + int64_t(w) * Q_pw + L.q_off;
        const int64_t n = L.cols * L.cap;
        for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
            const uint64_t h = mix64(base + uint64_t(i + 1) * kGamma);
            q[i] = __fsub_rn(__fmul_rn(float(h >> 40), 1.0f / 8388608.0f), 1.0f);
        }
    }
}


// The residual of one entry: m = fl32(M - sum_j P_j Q'_j), the sum formed
// as a product of column 0 then fused multiply-adds in column order -- in
// fp64 from the fp64 factors (T = double), or in fp32 from their fp32
// roundings, which are the P and Q the payload carries (T = float).  The
// residual pass and the lazy step's first pass form it identically.
// qv[j]: the factor Q' at this entry's column.
template <class T>
__device__ __forceinline__ float ps_unproject_v(float M, const T* pr, const T* qv, int r) {
    if constexpr (std::is_same<T, double>::value) {
        double mh = __dmul_rn(pr[0], qv[0]);
#pragma unroll
        for (int j = 1; j < kMaxRank; ++j)
            if (j < r) mh = __fma_rn(pr[j], qv[j], mh);
        return __double2float_rn(__dsub_rn(double(M), mh));
    } else {
        float mh = __fmul_rn(pr[0], qv[0]);
#pragma unroll
        for (int j = 1; j < kMaxRank; ++j)
            if (j < r) mh = __fmaf_rn(pr[j], qv[j], mh);
        return __fsub_rn(M, mh);
    }
}

template <class T>
__device__ __forceinline__ float ps_unproject(float M, const T* pr, const T (*qd)[kPsCB], int c,
                                              int r) {
    T qv[kMaxRank];
#pragma unroll
    for (int j = 0; j < kMaxRank; ++j) qv[j] = j < r ? qd[j][c] : T(0);
    return ps_unproject_v<T>(M, pr, qv, r);
}

// Four neighbouring shared-memory entries p[0..3] (16-byte aligned for
// float, 32-byte for double) in vector loads.
template <class T>
__device__ __forceinline__ void lds4(const T* p, T (&o)[4]) {
    if constexpr (std::is_same<T, double>::value) {
        const double2 a = *reinterpret_cast<const double2*>(p);
        const double2 b = *reinterpret_cast<const double2*>(p + 2);
        o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    } else {
        const float4 a = *reinterpret_cast<const float4*>(p);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    }
}

// One row of a M Q tile (cw columns from c0 of one 16-row block): M formed,
// optionally from the lazy residual, and written back; returns the row's
// partial P over the columns in acc (this lane's share, fp64).  The products
// in T (double or float); qs / qdp / pr hold the factors in T.  Full warp.
template <bool kLazy, class T>
__device__ __forceinline__ void ps_mq_row(const float* __restrict__ g, float* __restrict__ m,
                                          bool vec, int cw, float eta, int r, int rp,
                                          const T* pr, const T (*qs)[kPsCB],
                                          const T (*qdp)[kPsCB], double* acc) {
    const int lane = threadIdx.x & 31;
    T a[kMaxRank] = {T(0), T(0), T(0), T(0)};
    auto take = [&](float x, int c) {
#pragma unroll
        for (int j = 0; j < kMaxRank; ++j)
            if (j < r) {
                if constexpr (std::is_same<T, double>::value) a[j] = __fma_rn(double(x), qs[j][c], a[j]);
                else a[j] = __fmaf_rn(x, qs[j][c], a[j]);
            }
    };
    if (vec) {
        for (int c = lane * 4; c < cw; c += 128) {
            const float4 gg = ld_stream4(g + c);
            float4 mm = *reinterpret_cast<const float4*>(m + c);
            if (kLazy && rp > 0) {
                T qv[4][kMaxRank];  // qv[column][j], from vector loads of each factor column
#pragma unroll
                for (int j = 0; j < kMaxRank; ++j) {
                    T t4[4] = {T(0), T(0), T(0), T(0)};
                    if (j < rp) lds4<T>(&qdp[j][c], t4);
#pragma unroll
                    for (int i = 0; i < 4; ++i) qv[i][j] = t4[i];
                }
                mm.x = ps_unproject_v<T>(mm.x, pr, qv[0], rp);
                mm.y = ps_unproject_v<T>(mm.y, pr, qv[1], rp);
                mm.z = ps_unproject_v<T>(mm.z, pr, qv[2], rp);
                mm.w = ps_unproject_v<T>(mm.w, pr, qv[3], rp);
            }
            float4 x;
            x.x = residual(mm.x, eta, gg.x);
            x.y = residual(mm.y, eta, gg.y);
            x.z = residual(mm.z, eta, gg.z);
            x.w = residual(mm.w, eta, gg.w);
            *reinterpret_cast<float4*>(m + c) = x;
#pragma unroll
            for (int j = 0; j < kMaxRank; ++j)
                if (j < r) {
                    T q4[4];
                    lds4<T>(&qs[j][c], q4);
                    if constexpr (std::is_same<T, double>::value) {
                        a[j] = __fma_rn(double(x.x), q4[0], a[j]);
                        a[j] = __fma_rn(double(x.y), q4[1], a[j]);
                        a[j] = __fma_rn(double(x.z), q4[2], a[j]);
                        a[j] = __fma_rn(double(x.w), q4[3], a[j]);
                    } else {
                        a[j] = __fmaf_rn(x.x, q4[0], a[j]);
                        a[j] = __fmaf_rn(x.y, q4[1], a[j]);
                        a[j] = __fmaf_rn(x.z, q4[2], a[j]);
                        a[j] = __fmaf_rn(x.w, q4[3], a[j]);
                    }
                }
        }
    } else {
        for (int c = lane; c < cw; c += 32) {
            float mv = m[c];
            if (kLazy && rp > 0) mv = ps_unproject<T>(mv, pr, qdp, c, rp);
            const float x = residual(mv, eta, __ldcs(g + c));
            m[c] = x;
            take(x, c);
        }
    }
#pragma unroll
    for (int j = 0; j < kMaxRank; ++j) acc[j] = double(a[j]);
}

// Stage n entries of a rows x cap (row stride cap) factor, columns 0..rc-1,
// into dst[j][i] as T (double from fp64, or its fp32 rounding).
template <class T, class S>
__device__ __forceinline__ void ps_stage(T (*dst)[kPsCB], const S* src, int n, int rc,
                                         int cap) {
    for (int c = threadIdx.x; c < n; c += blockDim.x) {
        const S* x = src + int64_t(c) * cap;
#pragma unroll
        for (int j = 0; j < kMaxRank; ++j)
            if (j < rc) dst[j][c] = T(x[j]);
    }
}

// Rows x rc entries (row stride cap) into dst[row][j] as T.
template <class T, class S>
__device__ __forceinline__ void ps_stage_rows(T (*dst)[kMaxRank], const S* src, int rows, int rc,
                                              int cap) {
    for (int row = threadIdx.x; row < rows; row += blockDim.x) {
        const S* x = src + int64_t(row) * cap;
#pragma unroll
        for (int j = 0; j < kMaxRank; ++j)
            if (j < rc) dst[row][j] = T(x[j]);
    }
}

template <class T>
constexpr size_t ps_mq_smem(bool lazy) {
    return lazy ? sizeof(T) * (2 * kMaxRank * kPsCB + kPsRB * kMaxRank)
                : sizeof(T) * kMaxRank * kPsCB;
}
constexpr size_t kPsResidSmem = sizeof(double) * (kMaxRank * kPsCB + kPsRB * kMaxRank) +
                                sizeof(float) * (kMaxRank * kPsCB + kPsRB * kMaxRank);

template <class T>
constexpr const char* ps_prec_name(const char* d, const char* f) {
    return std::is_same<T, double>::value ? d : f;
}

// ---- phase 1: M = m + eta*g (written back), partial P = M Q -------------------------------
// Products in the layer's precision (kPsExactMax), sums across lanes and
// chunks in fp64.
// kLazy: the memory holds the previous step's M, the workspace that step's
// fp64 orthonormal P and Q' over lazy_rank[w][l] columns (0: the memory holds
// the residual itself); the residual m is formed on the fly, entry by entry
// as the residual pass would have formed it, so the results are the eager
// step's bit for bit without that pass's read and write of M.
template <bool kLazy, class T>
__global__ void __launch_bounds__(256, std::is_same<T, float>::value ? 5 : 4) ps_mq_kernel(
    const DevLayer* __restrict__ layers, const PsLayer* __restrict__ ps,
    const int4* __restrict__ tiles, int32_t ntiles, int32_t W, int64_t N, int64_t Q_pw,
    int64_t ppart_pw, const float* __restrict__ grad, float* __restrict__ mem, float eta,
    const int32_t* __restrict__ k_or_rank, const float* __restrict__ Q, double* __restrict__ ppart,
    int32_t* __restrict__ status, const double* __restrict__ pdw, int64_t pd_pw,
    const double* __restrict__ qdw, int32_t L_all, const int32_t* __restrict__ lazy_rank) {
    grid_dependency_sync();
    // dynamic shared memory (ps_mq_smem bytes)
    extern __shared__ __align__(16) double ps_dyn[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int64_t u = blockIdx.x; u < int64_t(ntiles) * W; u += gridDim.x) {
        const int w = int(u / ntiles);
        const int4 d = tiles[u % ntiles];
        const DevLayer L = layers[d.x];
        const PsLayer X = ps[d.x];
        const int r = ps_rank(L, k_or_rank, d.x);
        if (r == 0) continue;
        const int cap = L.cap;
        // columns of the previous step's factors to take off (lazy only)
        int rp = 0;
        if (kLazy) {
            rp = lazy_rank[int64_t(w) * L_all + d.x];
            rp = (rp >= 1 && rp <= cap) ? rp : 0;
        }
        const int64_t C = L.cols, R = L.rows;
        const int64_t c0 = int64_t(d.z) * kPsCB;
        const int cw = int(min64(kPsCB, C - c0));
        const int64_t r0 = d.y;
        const int rh = d.w;
        const float* q = Q + int64_t(w) * Q_pw + L.q_off + c0 * cap;
        // shared memory: the warm start Q, then (lazy) the previous Q' and
        // the previous P rows, in the layer's precision T
        {
            T (*qs)[kPsCB] = reinterpret_cast<T (*)[kPsCB]>(ps_dyn);
            T (*qdp)[kPsCB] = qs + kMaxRank;
            T (*prow)[kMaxRank] = reinterpret_cast<T (*)[kMaxRank]>(qdp + kMaxRank);
            ps_stage<T>(qs, q, cw, r, cap);
            if (kLazy && rp > 0) {
                ps_stage<T>(qdp, qdw + int64_t(w) * Q_pw + L.q_off + c0 * cap, cw, rp, cap);
                ps_stage_rows<T>(prow, pdw + int64_t(w) * pd_pw + X.pd_off + r0 * cap, rh, rp,
                                 cap);
            }
            __syncthreads();
            for (int row = warp; row < rh; row += blockDim.x >> 5) {
                const int64_t e = int64_t(w) * N + L.offset + (r0 + row) * C + c0;
                T pr[kMaxRank] = {T(0), T(0), T(0), T(0)};
                if (kLazy && rp > 0) {
#pragma unroll
                    for (int j = 0; j < kMaxRank; ++j) pr[j] = j < rp ? prow[row][j] : T(0);
                }
                double acc[kMaxRank];
                ps_mq_row<kLazy, T>(grad + e, mem + e, ((e & 3) == 0) && ((cw & 3) == 0), cw, eta,
                                    r, rp, pr, qs, qdp, acc);
                // a NaN or infinite M makes its row's products non-finite
                flag_nonfinite(!(fabs(acc[0]) <= 1.0e300), status);
#pragma unroll
                for (int j = 0; j < kMaxRank; ++j) acc[j] = warp_sum(acc[j]);
                if (lane < r) {
                    double a = acc[0];
                    if (lane == 1) a = acc[1];
                    if (lane == 2) a = acc[2];
                    if (lane == 3) a = acc[3];
                    ppart[int64_t(w) * ppart_pw + X.ppart_off + (int64_t(d.z) * R + r0 + row) * cap + lane] = a;
                }
            }
        }
        __syncthreads();
    }
}


// Entry (row, j) of P: the partials of nsum workers x nch column chunks
// added in fp64 in worker, then chunk order; kB partials are in flight
// ahead of their adds.
__device__ __forceinline__ double ps_sum_partials(const double* pp, int nsum, int64_t ppart_pw,
                                                  int nch, int64_t R, int cap, int64_t row,
                                                  int j) {
    constexpr int kB = 8;
    const int nt = nsum * nch;
    auto part = [&](int i) {
        const int ws = i / nch, ch = i - ws * nch;
        return __ldcg(pp + int64_t(ws) * ppart_pw + (int64_t(ch) * R + row) * cap + j);
    };
    double s = 0.0;
    int i = 0;
    for (; i + kB <= nt; i += kB) {
        double v[kB];
#pragma unroll
        for (int b = 0; b < kB; ++b) v[b] = part(i + b);
#pragma unroll
        for (int b = 0; b < kB; ++b) s += v[b];
    }
    for (; i < nt; ++i) s += part(i);
    return s;
}

// ---- orthonormalise P (one CTA per matrix) ----------------------------------------------
__device__ __forceinline__ double block_sum_d(double x, double* s_red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    x = warp_sum(x);
    if (lane == 0) s_red[warp] = x;
    __syncthreads();
    double t = 0.0;
    for (int i = 0; i < nw; ++i) t += s_red[i];
    __syncthreads();
    return t;
}

// Column passes of the Gram-Schmidt over this thread's rows (threadIdx.x,
// + blockDim.x, ...), in row order, with kU rows' loads issued ahead of their
// arithmetic.  ps_col_dot: sum of p_i * p_j; ps_col_axpy: p_j -= d p_i;
// ps_col_scale: p_j = p_j / nu (0 when nu is 0).
constexpr int kPsOrthThreads = 1024;

__device__ __forceinline__ double ps_col_dot(const double* pd, int64_t R, int cap, int i, int j) {
    constexpr int kU = 4;
    const int64_t B = blockDim.x;
    double part = 0.0;
    int64_t row = threadIdx.x;
    for (; row + (kU - 1) * B < R; row += kU * B) {
        double a[kU], b[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            a[u] = pd[(row + u * B) * cap + i];
            b[u] = pd[(row + u * B) * cap + j];
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) part += a[u] * b[u];
    }
    for (; row < R; row += B) part += pd[row * cap + i] * pd[row * cap + j];
    return part;
}

__device__ __forceinline__ void ps_col_axpy(double* pd, int64_t R, int cap, int i, int j,
                                            double d) {
    constexpr int kU = 4;
    const int64_t B = blockDim.x;
    int64_t row = threadIdx.x;
    for (; row + (kU - 1) * B < R; row += kU * B) {
        double a[kU], b[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            a[u] = pd[(row + u * B) * cap + i];
            b[u] = pd[(row + u * B) * cap + j];
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) pd[(row + u * B) * cap + j] = b[u] - d * a[u];
    }
    for (; row < R; row += B) pd[row * cap + j] -= d * pd[row * cap + i];
}

__device__ __forceinline__ void ps_col_scale(double* pd, int64_t R, int cap, int j, double nu) {
    constexpr int kU = 4;
    const int64_t B = blockDim.x;
    int64_t row = threadIdx.x;
    for (; row + (kU - 1) * B < R; row += kU * B) {
        double b[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) b[u] = pd[(row + u * B) * cap + j];
#pragma unroll
        for (int u = 0; u < kU; ++u) pd[(row + u * B) * cap + j] = nu > 0.0 ? b[u] / nu : 0.0;
    }
    for (; row < R; row += B) pd[row * cap + j] = nu > 0.0 ? pd[row * cap + j] / nu : 0.0;
}

// W outputs (one P per output); output w sums the partial P of workers
// w*nsum ... w*nsum + nsum - 1 in worker order (nsum = 1: independent
// replicas; W = 1, nsum = all workers: the data-parallel step).
__global__ void __launch_bounds__(kPsOrthThreads) ps_orth_kernel(
    const DevLayer* __restrict__ layers, const PsLayer* __restrict__ ps,
    const int32_t* __restrict__ ps_layers, int32_t nps, int32_t W, int32_t nsum, int64_t P_pw,
    int64_t ppart_pw,
    int64_t pd_pw, const int32_t* __restrict__ k_or_rank, const double* __restrict__ ppart,
    double* __restrict__ pdw, float* __restrict__ P, int32_t* __restrict__ status,
    int32_t ntall, int32_t* __restrict__ tdone, int32_t L_all, int32_t* __restrict__ lazy_rank) {
    grid_dependency_sync();
    __shared__ double s_red[32];
    for (int64_t u = blockIdx.x; u < int64_t(nps) * W; u += gridDim.x) {
        const int w = int(u / nps);
        const int32_t l = ps_layers[u % nps];
        const DevLayer L = layers[l];
        const PsLayer X = ps[l];
        const int r = ps_rank(L, k_or_rank, l);
        if (r == 0) {
            // a skipped layer keeps its memory, and in the lazy step its record
            if (threadIdx.x == 0) set_status(status, GCE_STATUS_K_RANGE);
            continue;
        }
        // the lazy step: the memory will hold M, P and Q this step's factors
        // (every M Q tile has read the previous record by now)
        if (lazy_rank && threadIdx.x == 0) lazy_rank[int64_t(w) * L_all + l] = r;
        if (X.tall >= 0) {  // orthonormalised by the multi-block kernel below
            if (threadIdx.x == 0) tdone[int64_t(w) * ntall + X.tall] = 0;
            continue;
        }
        const int cap = L.cap;
        const int64_t R = L.rows;
        const double* pp = ppart + int64_t(w) * nsum * ppart_pw + X.ppart_off;
        double* pd = pdw + int64_t(w) * pd_pw + X.pd_off;
        for (int64_t i = threadIdx.x; i < R * r; i += blockDim.x) {
            const int64_t row = i / r;
            const int j = int(i - row * r);
            pd[row * cap + j] = ps_sum_partials(pp, nsum, ppart_pw, X.nch1, R, cap, row, j);
        }
        __syncthreads();
        for (int j = 0; j < r; ++j) {
            for (int i = 0; i < j; ++i) {
                const double dot = block_sum_d(ps_col_dot(pd, R, cap, i, j), s_red);
                ps_col_axpy(pd, R, cap, i, j, dot);
                __syncthreads();
            }
            const double nu = sqrt(block_sum_d(ps_col_dot(pd, R, cap, j, j), s_red));
            ps_col_scale(pd, R, cap, j, nu);
            __syncthreads();
        }
        float* p = P + int64_t(w) * P_pw + L.p_off;
        for (int64_t i = threadIdx.x; i < R * r; i += blockDim.x) {
            const int64_t row = i / r;
            const int j = int(i - row * r);
            p[row * cap + j] = float(pd[row * cap + j]);
        }
        __syncthreads();
    }
}

// ---- orthonormalise tall P over many blocks ---------------------------------------------
// The same modified Gram-Schmidt, one launch per step: a launch first applies
// the previous step's update to its 256-row chunk (p_j -= d p_i, or
// p_j /= ||p_j||), then forms its chunk's part of the next dot product; the
// last block to finish adds the parts in chunk order (fixed, so the result is
// deterministic) and leaves the scalar for the next launch.
struct PsOrthOp {
    int8_t init;        // first launch: sum the partial P into fp64
    int8_t apply;       // 0 none, 1 subtract, 2 scale
    int8_t ai, aj;      // apply: p_aj -= d * p_ai, or p_aj /= sqrt(nn)
    int8_t reduce;      // 1: form p_ri . p_rj
    int8_t ri, rj;
    int8_t final_;      // last launch: write P in fp32
};

__global__ void __launch_bounds__(256) ps_orth_tall_kernel(
    PsOrthOp op, const DevLayer* __restrict__ layers, const PsLayer* __restrict__ ps,
    const int2* __restrict__ units, int32_t nunits, int32_t W, int32_t nsum, int64_t P_pw,
    int64_t ppart_pw, int64_t pd_pw, int32_t ntall, int32_t nparts,
    const int32_t* __restrict__ k_or_rank,
    const double* __restrict__ ppart, double* __restrict__ pdw, double* __restrict__ tparts,
    double* __restrict__ tscal, int32_t* __restrict__ tdone, float* __restrict__ P) {
    grid_dependency_sync();
    __shared__ double s_red[8];
    __shared__ int s_last;
    for (int64_t u = blockIdx.x; u < int64_t(nunits) * W; u += gridDim.x) {
        const int w = int(u / nunits);
        const int2 d = units[u % nunits];
        const DevLayer L = layers[d.x];
        const PsLayer X = ps[d.x];
        const int r = ps_rank(L, k_or_rank, d.x);
        if (r == 0) continue;
        const int cap = L.cap;
        const int64_t R = L.rows;
        const int64_t r0 = int64_t(d.y) * kPsOrthChunk;
        const int64_t r1 = min64(r0 + kPsOrthChunk, R);
        double* pd = pdw + int64_t(w) * pd_pw + X.pd_off;
        double* scal = tscal + int64_t(w) * ntall + X.tall;
        if (op.init) {
            const double* pp = ppart + int64_t(w) * nsum * ppart_pw + X.ppart_off;
            for (int64_t row = r0 + threadIdx.x; row < r1; row += blockDim.x)
                for (int j = 0; j < r; ++j)
                    pd[row * cap + j] = ps_sum_partials(pp, nsum, ppart_pw, X.nch1, R, cap, row, j);
        }
        if (op.apply && op.aj < r) {
            const double sv = *scal;
            if (op.apply == 1) {
                for (int64_t row = r0 + threadIdx.x; row < r1; row += blockDim.x)
                    pd[row * cap + op.aj] -= sv * pd[row * cap + op.ai];
            } else {
                const double nu = sqrt(sv);
                for (int64_t row = r0 + threadIdx.x; row < r1; row += blockDim.x)
                    pd[row * cap + op.aj] = nu > 0.0 ? pd[row * cap + op.aj] / nu : 0.0;
            }
        }
        if (op.reduce && op.rj < r) {
            double part = 0.0;
            for (int64_t row = r0 + threadIdx.x; row < r1; row += blockDim.x)
                part += pd[row * cap + op.ri] * pd[row * cap + op.rj];
            part = warp_sum(part);
            if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = part;
            __syncthreads();
            double* parts = tparts + int64_t(w) * nparts + X.part_off;
            if (threadIdx.x == 0) {
                double tsum = 0.0;
                for (int i = 0; i < int(blockDim.x >> 5); ++i) tsum += s_red[i];
                parts[d.y] = tsum;
                __threadfence();
                s_last = atomicAdd(&tdone[int64_t(w) * ntall + X.tall], 1) == X.nchunk - 1;
            }
            __syncthreads();
            if (s_last && threadIdx.x == 0) {
                __threadfence();
                // chunk order; eight parts in flight ahead of their adds
                double s = 0.0;
                int c = 0;
                for (; c + 8 <= X.nchunk; c += 8) {
                    double v[8];
#pragma unroll
                    for (int b = 0; b < 8; ++b) v[b] = __ldcg(parts + c + b);
#pragma unroll
                    for (int b = 0; b < 8; ++b) s += v[b];
                }
                for (; c < X.nchunk; ++c) s += __ldcg(parts + c);
                *scal = s;
                tdone[int64_t(w) * ntall + X.tall] = 0;  // ready for the next launch
            }
        }
        if (op.final_) {
            float* p = P + int64_t(w) * P_pw + L.p_off;
            for (int64_t row = r0 + threadIdx.x; row < r1; row += blockDim.x)
                for (int j = 0; j < r; ++j) p[row * cap + j] = float(pd[row * cap + j]);
        }
        __syncthreads();
    }
}

// the launch sequence for P with up to `cap` columns
static std::vector<PsOrthOp> ps_orth_ops(int cap) {
    std::vector<PsOrthOp> ops;
    PsOrthOp cur{};
    cur.init = 1;
    auto push_reduce = [&](int i, int j) {
        cur.reduce = 1;
        cur.ri = int8_t(i);
        cur.rj = int8_t(j);
        ops.push_back(cur);
        cur = PsOrthOp{};
    };
    for (int j = 0; j < cap; ++j) {
        for (int i = 0; i < j; ++i) {
            push_reduce(i, j);
            cur.apply = 1;
            cur.ai = int8_t(i);
            cur.aj = int8_t(j);
        }
        push_reduce(j, j);
        cur.apply = 2;
        cur.ai = cur.aj = int8_t(j);
    }
    cur.final_ = 1;
    ops.push_back(cur);
    return ops;
}

// ---- phase 3: partial Q = M^T P over row blocks ----------------------------------------------
// From the orthonormal P of the workspace: products in the layer's
// precision (fp64, or fp32 from the P the payload carries), the partial of
// each row block (PsLayer::rb3 rows) stored in fp64.
template <class T>
__global__ void __launch_bounds__(256, std::is_same<T, float>::value ? 6 : 4) ps_mtp_kernel(
    const DevLayer* __restrict__ layers, const PsLayer* __restrict__ ps,
    const int4* __restrict__ tiles, int32_t ntiles, int32_t W, int64_t N, int64_t pd_pw,
    int64_t qpart_pw, const float* __restrict__ mem, const int32_t* __restrict__ k_or_rank,
    const double* __restrict__ pdw, double* __restrict__ qpart) {
    grid_dependency_sync();
    __shared__ double prow_d[kPsRB3][kMaxRank];
    const int tid = threadIdx.x;
    for (int64_t u = blockIdx.x; u < int64_t(ntiles) * W; u += gridDim.x) {
        const int w = int(u / ntiles);
        const int4 d = tiles[u % ntiles];
        const DevLayer L = layers[d.x];
        const PsLayer X = ps[d.x];
        const int r = ps_rank(L, k_or_rank, d.x);
        if (r == 0) continue;
        const int cap = L.cap;
        const int64_t C = L.cols;
        const int64_t r0 = int64_t(d.y) * X.rb3;
        const int rh = int(min64(X.rb3, L.rows - r0));
        const int64_t c0 = int64_t(d.z) * kPsCB;
        const int cw = int(min64(kPsCB, C - c0));
        const double* p = pdw + int64_t(w) * pd_pw + X.pd_off + r0 * cap;
        const int cc = tid * 4;
        const int64_t ebase = int64_t(w) * N + L.offset + r0 * C + c0;
        const bool vec = ((ebase & 3) == 0) && ((C & 3) == 0) && (cc + 3 < cw);
        double* out = qpart + int64_t(w) * qpart_pw + X.qpart_off + (int64_t(d.y) * C + c0 + cc) * cap;
        {
            T (*prow)[kMaxRank] = reinterpret_cast<T (*)[kMaxRank]>(&prow_d[0][0]);
            for (int i = tid; i < rh * kMaxRank; i += blockDim.x) {
                const int row = i / kMaxRank, j = i % kMaxRank;
                prow[row][j] = j < r ? T(p[int64_t(row) * cap + j]) : T(0);
            }
            __syncthreads();
            T acc[4][kMaxRank];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int j = 0; j < kMaxRank; ++j) acc[q][j] = T(0);
            if (cc < cw) {
                auto fma_row = [&](const float (&x)[4], int row) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
#pragma unroll
                        for (int j = 0; j < kMaxRank; ++j)
                            if (j < r) {
                                if constexpr (std::is_same<T, double>::value)
                                    acc[q][j] = __fma_rn(double(x[q]), prow[row][j], acc[q][j]);
                                else
                                    acc[q][j] = __fmaf_rn(x[q], prow[row][j], acc[q][j]);
                            }
                };
                int row = 0;
                if (vec) {
                    // kB rows' loads in flight before their products (rows in order)
                    constexpr int kB = 8;
                    for (; row + kB <= rh; row += kB) {
                        float4 mm[kB];
#pragma unroll
                        for (int b = 0; b < kB; ++b)
                            mm[b] = __ldg(reinterpret_cast<const float4*>(mem + ebase +
                                                                          int64_t(row + b) * C + cc));
#pragma unroll
                        for (int b = 0; b < kB; ++b) {
                            const float x[4] = {mm[b].x, mm[b].y, mm[b].z, mm[b].w};
                            fma_row(x, row + b);
                        }
                    }
                }
                for (; row < rh; ++row) {
                    const float* m = mem + ebase + int64_t(row) * C + cc;
                    float x[4];
                    if (vec) {
                        const float4 mm = *reinterpret_cast<const float4*>(m);
                        x[0] = mm.x; x[1] = mm.y; x[2] = mm.z; x[3] = mm.w;
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) x[q] = (cc + q < cw) ? m[q] : 0.0f;
                    }
                    fma_row(x, row);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (cc + q < cw)
#pragma unroll
                        for (int j = 0; j < kMaxRank; ++j)
                            if (j < r) out[q * cap + j] = double(acc[q][j]);
            }
        }
        __syncthreads();
    }
}

// ---- Q = sum of the row-block partials (fp64, block order) ----------------------------------
// Q' in fp64 to qd (stride Q_pw per worker) and rounded to fp32 to Q.  A layer
// of kPsQSplit or more row blocks sums them as four contiguous quarters, each
// in block order, added in order (a fixed order, the same every call).
// kMean (the data-parallel step): every worker's Q_w goes to Q (stride
// Q_pw, fp32) and qd (fp64), and their mean -- fp32 sum of the rounded Q_w in
// worker order from +0, times inv_w -- to qmean, one tile per block for all W
// workers.
template <bool kMean>
__global__ void __launch_bounds__(256) ps_qred_kernel(
    const DevLayer* __restrict__ layers, const PsLayer* __restrict__ ps,
    const int4* __restrict__ tiles, int32_t ntiles, int32_t W, int64_t Q_pw, int64_t qpart_pw,
    const int32_t* __restrict__ k_or_rank, const double* __restrict__ qpart,
    float* __restrict__ Q, double* __restrict__ qd, float* __restrict__ qmean, float inv_w) {
    grid_dependency_sync();
    const int64_t nunits = kMean ? int64_t(ntiles) : int64_t(ntiles) * W;
    for (int64_t u = blockIdx.x; u < nunits; u += gridDim.x) {
        const int w = kMean ? 0 : int(u / ntiles);
        const int4 d = tiles[u % ntiles];
        const DevLayer L = layers[d.x];
        const PsLayer X = ps[d.x];
        const int r = ps_rank(L, k_or_rank, d.x);
        if (r == 0) continue;
        const int cap = L.cap;
        const int64_t C = L.cols;
        const int64_t c0 = d.y;
        const int cw = d.z;
        // G lanes per entry: with many row blocks, lane g of the group sums
        // the g-th contiguous quarter of them in block order and the group
        // adds the quarters in order; with few, one lane sums them all
        const int G = X.nrb3 >= kPsQSplit ? 4 : 1;
        const int nb = (X.nrb3 + G - 1) / G;
        const int n = cw * r * G;
        for (int i0 = 0; i0 < n; i0 += blockDim.x) {
            const int i = i0 + int(threadIdx.x);
            const bool act = i < n;
            const int item = i / G, g = i - item * G;
            const int64_t c = c0 + item / r;
            const int j = item % r;
            float mean = 0.0f;
            for (int wi = 0; wi < (kMean ? W : 1); ++wi) {
                const int ww = kMean ? wi : w;
                const double* qp = qpart + int64_t(ww) * qpart_pw + X.qpart_off;
                // block order; kB partials in flight ahead of their adds
                constexpr int kB = 8;
                const int64_t stride = C * cap;
                const double* x = qp + c * cap + j;
                const int rb0 = g * nb, rb1 = act ? min(X.nrb3, rb0 + nb) : rb0;
                double s = 0.0;
                int rb = rb0;
                for (; rb + kB <= rb1; rb += kB) {
                    double v[kB];
#pragma unroll
                    for (int b = 0; b < kB; ++b) v[b] = __ldcg(x + int64_t(rb + b) * stride);
#pragma unroll
                    for (int b = 0; b < kB; ++b) s += v[b];
                }
                for (; rb < rb1; ++rb) s += __ldcg(x + int64_t(rb) * stride);
                if (G == 4) {  // the group's quarters, in order, into its first lane
                    const double s1 = __shfl_down_sync(kFull, s, 1);
                    const double s2 = __shfl_down_sync(kFull, s, 2);
                    const double s3 = __shfl_down_sync(kFull, s, 3);
                    s = ((s + s1) + s2) + s3;
                }
                if (act && g == 0) {
                    const float qv = float(s);
                    Q[int64_t(ww) * Q_pw + L.q_off + c * cap + j] = qv;
                    qd[int64_t(ww) * Q_pw + L.q_off + c * cap + j] = s;
                    if (kMean) mean = __fadd_rn(mean, qv);
                }
            }
            if (kMean && act && g == 0) qmean[L.q_off + c * cap + j] = __fmul_rn(mean, inv_w);
        }
    }
}

// ---- data-parallel DENSE layers: payload = mean of the workers' residuals ------------------
__global__ void __launch_bounds__(256) ps_dense_mean_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ dtile_layer,
    const int32_t* __restrict__ dtile_start, int32_t ntiles, int32_t W, int64_t N,
    const float* __restrict__ grad, float* __restrict__ mem, float eta, float inv_w,
    float* __restrict__ vals, int32_t* __restrict__ status) {
    grid_dependency_sync();
    bool bad = false;
    for (int32_t u = blockIdx.x; u < ntiles; u += gridDim.x) {
        const DevLayer L = layers[dtile_layer[u]];
        const int64_t s0 = dtile_start[u];
        const int64_t cnt = min64(int64_t(kDenseTile), L.n - s0);
        for (int64_t i = threadIdx.x; i < cnt; i += blockDim.x) {
            float s = 0.0f;
            for (int w = 0; w < W; ++w) {
                const int64_t e = int64_t(w) * N + L.offset + s0 + i;
                s = __fadd_rn(s, residual(mem[e], eta, __ldcs(grad + e)));
                mem[e] = 0.0f;
            }
            bad |= abs_key(s) >= kNonFiniteKey;
            vals[L.val_off + s0 + i] = __fmul_rn(s, inv_w);
        }
    }
    flag_nonfinite(bad, status);
}

// ---- the workers' means after an exchange between ranks ------------------------------------
// Q = fl(fl(sum_w Q_w) * inv_w) over W gathered rows of Q_w (worker order from
// +0, fp32), as the one-GPU data-parallel step forms its warm start.
__global__ void __launch_bounds__(256) ps_qmean_kernel(
    const DevLayer* __restrict__ layers, const int4* __restrict__ tiles, int32_t ntiles,
    int32_t W, int64_t Q_pw, const int32_t* __restrict__ k_or_rank, const float* __restrict__ Qw,
    float* __restrict__ Q, float inv_w) {
    grid_dependency_sync();
    for (int32_t u = blockIdx.x; u < ntiles; u += gridDim.x) {
        const int4 d = tiles[u];
        const DevLayer L = layers[d.x];
        const int r = ps_rank(L, k_or_rank, d.x);
        if (r == 0) continue;
        const int cap = L.cap;
        const int64_t c0 = d.y;
        const int cw = d.z;
        for (int i = threadIdx.x; i < cw * r; i += blockDim.x) {
            const int64_t o = L.q_off + (c0 + i / r) * cap + i % r;
            float sum = 0.0f;
            for (int w = 0; w < W; ++w) sum = __fadd_rn(sum, Qw[int64_t(w) * Q_pw + o]);
            Q[o] = __fmul_rn(sum, inv_w);
        }
    }
}

// DENSE layers: mean = fl(fl(sum_w v_w) * inv_w) over W gathered payload rows.
__global__ void __launch_bounds__(256) ps_vmean_kernel(
    const DevLayer* __restrict__ layers, const int32_t* __restrict__ dtile_layer,
    const int32_t* __restrict__ dtile_start, int32_t ntiles, int32_t W, int64_t vals_pw,
    const float* __restrict__ vals_all, float* __restrict__ vals, float inv_w) {
    grid_dependency_sync();
    for (int32_t u = blockIdx.x; u < ntiles; u += gridDim.x) {
        const DevLayer L = layers[dtile_layer[u]];
        const int64_t s0 = dtile_start[u];
        const int64_t cnt = min64(int64_t(kDenseTile), L.n - s0);
        for (int64_t i = threadIdx.x; i < cnt; i += blockDim.x) {
            float sum = 0.0f;
            for (int w = 0; w < W; ++w)
                sum = __fadd_rn(sum, vals_all[int64_t(w) * vals_pw + L.val_off + s0 + i]);
            vals[L.val_off + s0 + i] = __fmul_rn(sum, inv_w);
        }
    }
}

// ---- residual: m <- M - P Q^T, dense_out <- P Q^T ---------------------------------------------
// The memory from the workspace's factors in the layer's precision
// (ps_unproject); dense_out from the fp32 P and Q the payload carries, formed
// as the decoder forms it (product, then fp32 fused multiply-adds in column
// order), so dense_out is the decode.
// rank_wl (nullable): per (worker, layer) ranks [W][L_all] instead of
// k_or_rank -- the lazy step's record, for gce_materialize_memory.
template <class T>
__global__ void __launch_bounds__(256) ps_resid_kernel(
    const DevLayer* __restrict__ layers, const PsLayer* __restrict__ ps,
    const int4* __restrict__ tiles, int32_t ntiles, int32_t W, int64_t N, int64_t P_pw,
    int64_t Q_pw, int64_t pd_pw, const int32_t* __restrict__ k_or_rank,
    const float* __restrict__ P, const float* __restrict__ Q, const double* __restrict__ pdw,
    const double* __restrict__ qdw, float* __restrict__ mem, float* __restrict__ dense_out,
    const int32_t* __restrict__ rank_wl, int32_t L_all) {
    grid_dependency_sync();
    // dynamic shared memory (kPsResidSmem bytes)
    extern __shared__ __align__(16) double ps_dyn[];
    float (*qs)[kPsCB] =
        reinterpret_cast<float (*)[kPsCB]>(ps_dyn + kMaxRank * kPsCB + kPsRB * kMaxRank);
    float (*prow32)[kMaxRank] = reinterpret_cast<float (*)[kMaxRank]>(
        reinterpret_cast<float*>(qs) + kMaxRank * kPsCB);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int64_t u = blockIdx.x; u < int64_t(ntiles) * W; u += gridDim.x) {
        const int w = int(u / ntiles);
        const int4 d = tiles[u % ntiles];
        const DevLayer L = layers[d.x];
        const PsLayer X = ps[d.x];
        int r = 0;
        if (rank_wl) {
            r = rank_wl[int64_t(w) * L_all + d.x];
            r = (r >= 1 && r <= L.cap) ? r : 0;
        } else {
            r = ps_rank(L, k_or_rank, d.x);
        }
        if (r == 0) continue;
        const int cap = L.cap;
        const int64_t C = L.cols;
        const int64_t c0 = int64_t(d.z) * kPsCB;
        const int cw = int(min64(kPsCB, C - c0));
        const int64_t r0 = d.y;
        const int rh = d.w;
        if (dense_out) {
            ps_stage<float>(qs, Q + int64_t(w) * Q_pw + L.q_off + c0 * cap, cw, r, cap);
            ps_stage_rows<float>(prow32, P + int64_t(w) * P_pw + L.p_off + r0 * cap, rh, r, cap);
        }
        {
            T (*qd)[kPsCB] = reinterpret_cast<T (*)[kPsCB]>(ps_dyn);
            T (*prow)[kMaxRank] = reinterpret_cast<T (*)[kMaxRank]>(ps_dyn + kMaxRank * kPsCB);
            ps_stage<T>(qd, qdw + int64_t(w) * Q_pw + L.q_off + c0 * cap, cw, r, cap);
            ps_stage_rows<T>(prow, pdw + int64_t(w) * pd_pw + X.pd_off + r0 * cap, rh, r, cap);
            __syncthreads();
            for (int row = warp; row < rh; row += blockDim.x >> 5) {
                const int64_t e = int64_t(w) * N + L.offset + (r0 + row) * C + c0;
                float* m = mem + e;
                float* o = dense_out ? dense_out + e : nullptr;
                T pr[kMaxRank];
                float pr32[kMaxRank];
#pragma unroll
                for (int j = 0; j < kMaxRank; ++j) {
                    pr[j] = j < r ? prow[row][j] : T(0);
                    pr32[j] = (o && j < r) ? prow32[row][j] : 0.0f;
                }
                auto decoded = [&](int c) {
                    float mh = __fmul_rn(pr32[0], qs[0][c]);
#pragma unroll
                    for (int j = 1; j < kMaxRank; ++j)
                        if (j < r) mh = __fmaf_rn(pr32[j], qs[j][c], mh);
                    return mh;
                };
                if (((e & 3) == 0) && ((cw & 3) == 0)) {  // 16-byte rows: four columns a lane
                    // float4 of memory in flight per lane (fewer for the fp64 products)
                    constexpr int kU = std::is_same<T, double>::value ? 2 : 4;
                    for (int c0 = lane * 4; c0 < cw; c0 += 128 * kU) {
                        float4 mm[kU];
#pragma unroll
                        for (int u = 0; u < kU; ++u)
                            if (c0 + 128 * u < cw)
                                mm[u] = *reinterpret_cast<const float4*>(m + c0 + 128 * u);
#pragma unroll
                        for (int u = 0; u < kU; ++u) {
                            const int c = c0 + 128 * u;
                            if (c >= cw) break;
                            float4 mv = mm[u];
                            T qv[4][kMaxRank];
#pragma unroll
                            for (int j = 0; j < kMaxRank; ++j) {
                                T t4[4] = {T(0), T(0), T(0), T(0)};
                                if (j < r) lds4<T>(&qd[j][c], t4);
#pragma unroll
                                for (int i = 0; i < 4; ++i) qv[i][j] = t4[i];
                            }
                            mv.x = ps_unproject_v<T>(mv.x, pr, qv[0], r);
                            mv.y = ps_unproject_v<T>(mv.y, pr, qv[1], r);
                            mv.z = ps_unproject_v<T>(mv.z, pr, qv[2], r);
                            mv.w = ps_unproject_v<T>(mv.w, pr, qv[3], r);
                            __stcs(reinterpret_cast<float4*>(m + c), mv);
                            if (o)
                                __stcs(reinterpret_cast<float4*>(o + c),
                                       make_float4(decoded(c), decoded(c + 1), decoded(c + 2),
                                                   decoded(c + 3)));
                        }
                    }
                } else {
                    for (int c = lane; c < cw; c += 32) {
                        m[c] = ps_unproject<T>(m[c], pr, qd, c, r);
                        if (o) o[c] = decoded(c);
                    }
                }
            }
        }
        __syncthreads();
    }
}

// ---- decode of PowerSGD payloads: out = scale * sum_w P_w Q_w^T ---------------------------
// Per (16-row, 1024-column) tile, in 256-column quarters: the quarter's Q
// columns and the tile's P rows of every worker sit in shared memory, each
// thread owns one column and walks the 16 rows, so the output is written in
// full 128-byte lines.  Each entry is formed exactly as the element-wise
// decoder forms it (product, then fused multiply-adds in column order, then
// the workers summed in order from +0), so both give the same bits.
constexpr int kDcLrMaxW = 8;

template <bool kApply>
__global__ void __launch_bounds__(256) ps_decode_kernel(
    const DevLayer* __restrict__ layers, const int4* __restrict__ tiles, int32_t ntiles,
    int32_t W, int64_t P_pw, int64_t Q_pw, const int32_t* __restrict__ k_or_rank,
    const float* __restrict__ P, const float* __restrict__ Q, float scale,
    float* __restrict__ out) {
    grid_dependency_sync();
    __shared__ float qs[kDcLrMaxW][kMaxRank][256];
    __shared__ float prow[kDcLrMaxW][kPsRB][kMaxRank];
    const int tid = threadIdx.x;
    for (int32_t u = blockIdx.x; u < ntiles; u += gridDim.x) {
        const int4 d = tiles[u];
        const DevLayer L = layers[d.x];
        const int r = ps_rank(L, k_or_rank, d.x);
        const int cap = L.cap;
        const int64_t C = L.cols;
        const int64_t r0 = d.y;
        const int rh = d.w;
        const int64_t c0 = int64_t(d.z) * kPsCB;
        const int cw = int(min64(kPsCB, C - c0));
        for (int i = tid; i < W * rh; i += blockDim.x) {
            const int w = i / rh, rr = i - w * rh;
            const float* p = P + int64_t(w) * P_pw + L.p_off + (r0 + rr) * cap;
#pragma unroll
            for (int j = 0; j < kMaxRank; ++j) prow[w][rr][j] = j < r ? p[j] : 0.0f;
        }
        const bool rows16 = ((L.offset + r0 * C + c0) & 3) == 0 && (C & 3) == 0 && (cw & 3) == 0;
        if (W == 1 && rows16) {
            // one worker, 16-byte rows: a thread owns four neighbouring columns,
            // keeps their Q in registers and writes float4s down the 16 rows
            __syncthreads();
            const int cc = tid * 4;
            if (cc < cw) {
                float q[4][kMaxRank];
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < kMaxRank; ++j)
                        q[c][j] = j < r ? __ldg(Q + L.q_off + (c0 + cc + c) * cap + j) : 0.0f;
                float* o = out + L.offset + r0 * C + c0 + cc;
                for (int rr = 0; rr < rh; ++rr) {
                    float v[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float m = 0.0f;
                        if (r > 0) {
                            m = __fmul_rn(prow[0][rr][0], q[c][0]);
#pragma unroll
                            for (int j = 1; j < kMaxRank; ++j)
                                if (j < r) m = __fmaf_rn(prow[0][rr][j], q[c][j], m);
                        }
                        v[c] = __fadd_rn(0.0f, m);
                    }
                    float4* o4 = reinterpret_cast<float4*>(o + int64_t(rr) * C);
                    *o4 = dc_final4<kApply>(make_float4(v[0], v[1], v[2], v[3]), scale, o4);
                }
            }
            __syncthreads();
            continue;
        }
        for (int qb = 0; qb < cw; qb += 256) {
            __syncthreads();
            for (int i = tid; i < W * kMaxRank * 256; i += blockDim.x) {
                const int w = i / (kMaxRank * 256), j = (i / 256) % kMaxRank, c = i % 256;
                qs[w][j][c] = (j < r && qb + c < cw)
                                  ? Q[int64_t(w) * Q_pw + L.q_off + (c0 + qb + c) * cap + j]
                                  : 0.0f;
            }
            __syncthreads();
            const int c = qb + tid;
            if (c < cw) {
                float* o = out + L.offset + r0 * C + c0 + c;
                for (int rr = 0; rr < rh; ++rr) {
                    float s = 0.0f;
                    for (int w = 0; w < W; ++w) {
                        float m = 0.0f;
                        if (r > 0) {
                            m = __fmul_rn(prow[w][rr][0], qs[w][0][tid]);
                            for (int j = 1; j < r; ++j) m = __fmaf_rn(prow[w][rr][j], qs[w][j][tid], m);
                        }
                        s = __fadd_rn(s, m);
                    }
                    o[int64_t(rr) * C] = dc_final<kApply>(s, scale, o + int64_t(rr) * C);
                }
            }
        }
        __syncthreads();
    }
}

// PowerSGD layers of the decode; false: W too large, use the element-wise path
bool launch_lowrank_decode(const gce_table* t, int32_t W, const int32_t* k_or_rank, const float* P,
                           const float* Q, float scale, float* out, bool apply, cudaStream_t st) {
    if (W > kDcLrMaxW) return false;
    static const int r_dec = resident_blocks(ps_decode_kernel<false>, 256);
    static const int r_dec_apply = resident_blocks(ps_decode_kernel<true>, 256);
    if (t->ps1_ntiles > 0 && !apply)
        GCE_LAUNCH(ps_decode_kernel<false>, wave_grid(t->ps1_ntiles, 4, r_dec), 256, 0, st,
                   t->d_layers, t->d_ps1_tiles, t->ps1_ntiles, W, t->P_pw, t->Q_pw, k_or_rank, P,
                   Q, scale, out);
    if (t->ps1_ntiles > 0 && apply)
        GCE_LAUNCH(ps_decode_kernel<true>, wave_grid(t->ps1_ntiles, 4, r_dec_apply), 256, 0, st,
                   t->d_layers, t->d_ps1_tiles, t->ps1_ntiles, W, t->P_pw, t->Q_pw, k_or_rank, P,
                   Q, scale, out);
    return true;
}

// ---- launches over both precisions: the fp64-product layers' tiles come first ------------
template <bool kLazy, class T>
static void ps_launch_mq_part(const gce_table* t, const int4* tiles, int32_t n, int32_t W,
                              int64_t Q_pw, const float* grad, float* mem, float eta,
                              const int32_t* k_or_rank, const float* Q, double* ppart,
                              int32_t* status, const double* pd, int64_t pd_pw, const double* qd,
                              const int32_t* lazy_rank, cudaStream_t st) {
    if (n <= 0) return;
    static const int r = resident_blocks_smem(ps_mq_kernel<kLazy GCE_COMMA T>, 256,
                                              ps_mq_smem<T>(kLazy));
    GCE_LAUNCH_AS(kLazy ? ps_prec_name<T>("ps_mq_kernel<lazy,f64>", "ps_mq_kernel<lazy,f32>")
                        : ps_prec_name<T>("ps_mq_kernel<f64>", "ps_mq_kernel<f32>"),
                  ps_mq_kernel<kLazy GCE_COMMA T>, wave_grid(int64_t(n) * W, 8, r), 256,
                  ps_mq_smem<T>(kLazy), st, t->d_layers, static_cast<const PsLayer*>(t->d_ps),
                  tiles, n, W, t->N, Q_pw, t->ppart_pw, grad, mem, eta, k_or_rank, Q, ppart,
                  status, pd, pd_pw, qd, t->L, lazy_rank);
}

// M Q pass (and the memory's M) over every PowerSGD tile; Q_pw 0: one Q for
// every worker.  lazy_rank non-null: the lazy first pass.
static void ps_launch_mq(const gce_table* t, int32_t W, int64_t Q_pw, const float* grad,
                         float* mem, float eta, const int32_t* k_or_rank, const float* Q,
                         double* ppart, int32_t* status, const double* pd, int64_t pd_pw,
                         const double* qd, const int32_t* lazy_rank, cudaStream_t st) {
    const int32_t nx = t->ps1_nexact, nf = t->ps1_ntiles - nx;
    const int4* tx = t->d_ps1_tiles;
    const int4* tf = t->d_ps1_tiles + nx;
    if (lazy_rank) {
        ps_launch_mq_part<true, double>(t, tx, nx, W, Q_pw, grad, mem, eta, k_or_rank, Q, ppart,
                                        status, pd, pd_pw, qd, lazy_rank, st);
        ps_launch_mq_part<true, float>(t, tf, nf, W, Q_pw, grad, mem, eta, k_or_rank, Q, ppart,
                                       status, pd, pd_pw, qd, lazy_rank, st);
    } else {
        ps_launch_mq_part<false, double>(t, tx, nx, W, Q_pw, grad, mem, eta, k_or_rank, Q,
                                         ppart, status, pd, pd_pw, qd, lazy_rank, st);
        ps_launch_mq_part<false, float>(t, tf, nf, W, Q_pw, grad, mem, eta, k_or_rank, Q, ppart,
                                        status, pd, pd_pw, qd, lazy_rank, st);
    }
}

template <class T>
static void ps_launch_mtp_part(const gce_table* t, const int4* tiles, int32_t n, int32_t W,
                               int64_t pd_pw, const float* mem, const int32_t* k_or_rank,
                               const double* pd, double* qpart, cudaStream_t st) {
    if (n <= 0) return;
    static const int r = resident_blocks(ps_mtp_kernel<T>, 256);
    GCE_LAUNCH_AS(ps_prec_name<T>("ps_mtp_kernel<f64>", "ps_mtp_kernel<f32>"), ps_mtp_kernel<T>,
                  wave_grid(int64_t(n) * W, 8, r), 256, 0, st, t->d_layers,
                  static_cast<const PsLayer*>(t->d_ps), tiles, n, W, t->N, pd_pw, t->qpart_pw,
                  mem, k_or_rank, pd, qpart);
}

// partial Q = M^T P over every PowerSGD tile; pd_pw 0: one P for every worker
static void ps_launch_mtp(const gce_table* t, int32_t W, int64_t pd_pw, const float* mem,
                          const int32_t* k_or_rank, const double* pd, double* qpart,
                          cudaStream_t st) {
    const int32_t nx = t->ps3_nexact;
    ps_launch_mtp_part<double>(t, t->d_ps3_tiles, nx, W, pd_pw, mem, k_or_rank, pd, qpart, st);
    ps_launch_mtp_part<float>(t, t->d_ps3_tiles + nx, t->ps3_ntiles - nx, W, pd_pw, mem,
                              k_or_rank, pd, qpart, st);
}

template <class T>
static void ps_launch_resid_part(const gce_table* t, const int4* tiles, int32_t n, int32_t W,
                                 int64_t P_pw, int64_t Q_pw, int64_t pd_pw,
                                 const int32_t* k_or_rank, const float* P, const float* Q,
                                 const double* pd, const double* qd, float* mem,
                                 float* dense_out, const int32_t* rank_wl, cudaStream_t st) {
    if (n <= 0) return;
    static const int r = resident_blocks_smem(ps_resid_kernel<T>, 256, kPsResidSmem);
    GCE_LAUNCH_AS(ps_prec_name<T>("ps_resid_kernel<f64>", "ps_resid_kernel<f32>"),
                  ps_resid_kernel<T>, wave_grid(int64_t(n) * W, 8, r), 256, kPsResidSmem, st,
                  t->d_layers, static_cast<const PsLayer*>(t->d_ps), tiles, n, W, t->N, P_pw,
                  Q_pw, pd_pw, k_or_rank, P, Q, pd, qd, mem, dense_out, rank_wl, t->L);
}

// m <- M - P Q^T over every PowerSGD tile (rank_wl: the lazy record)
static void ps_launch_resid(const gce_table* t, int32_t W, int64_t P_pw, int64_t Q_pw,
                            int64_t pd_pw, const int32_t* k_or_rank, const float* P,
                            const float* Q, const double* pd, const double* qd, float* mem,
                            float* dense_out, const int32_t* rank_wl, cudaStream_t st) {
    const int32_t nx = t->ps1_nexact;
    ps_launch_resid_part<double>(t, t->d_ps1_tiles, nx, W, P_pw, Q_pw, pd_pw, k_or_rank, P, Q,
                                 pd, qd, mem, dense_out, rank_wl, st);
    ps_launch_resid_part<float>(t, t->d_ps1_tiles + nx, t->ps1_ntiles - nx, W, P_pw, Q_pw,
                                pd_pw, k_or_rank, P, Q, pd, qd, mem, dense_out, rank_wl, st);
}

}  // namespace gce

using namespace gce;

extern "C" int powersgd_init_q(const gce_table* t, int32_t W, uint64_t seed, float* Q, void* stream) {
    if (!t || W < 1) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_POWERSGD && t->ckind != -1) return GCE_ERR_KIND;
    if (t->nps == 0) return GCE_OK;
    if (!Q || !aligned16(Q)) return GCE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    static const int r_init = resident_blocks(ps_init_q_kernel, 256);
    GCE_LAUNCH(ps_init_q_kernel, wave_grid(int64_t(t->nps) * W, 4, r_init), 256, 0, st, t->d_layers,
               t->d_ps_layers, t->nps, W, t->Q_pw, seed, Q);
    return check_launch();
}

static int ps_step(const gce_table* t, int32_t W, const float* grad, float* mem, float eta,
                   const int32_t* k_or_rank, float* P, float* Q, float* vals, float* dense_out,
                   int32_t* lazy_rank, void* ws, size_t ws_bytes, void* stream) {
    if (!t || W < 1 || !grad || !mem || !ws) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_POWERSGD && t->ckind != -1) return GCE_ERR_KIND;
    if (!aligned16(grad) || !aligned16(mem) || !aligned16(ws)) return GCE_ERR_ARG;
    if (t->nps > 0 && (!P || !Q || !aligned16(P) || !aligned16(Q))) return GCE_ERR_ARG;
    if (dense_out && !aligned16(dense_out)) return GCE_ERR_ARG;
    if (k_or_rank && (reinterpret_cast<uintptr_t>(k_or_rank) & 3)) return GCE_ERR_ARG;
    const PsWs lay = ps_layout(t, W);
    if (ws_bytes < lay.total) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = static_cast<int32_t*>(ws);
    if (t->nps > 0) {
        double* ppart = at<double>(ws, lay.ppart);
        double* pd = at<double>(ws, lay.pd);
        double* qpart = at<double>(ws, lay.qpart);
        double* qd = at<double>(ws, lay.qd);
        const PsLayer* ps = static_cast<const PsLayer*>(t->d_ps);
        static const int r_orth = resident_blocks(ps_orth_kernel, kPsOrthThreads);
        static const int r_tall = resident_blocks(ps_orth_tall_kernel, 256);
        static const int r_qred = resident_blocks(ps_qred_kernel<false>, 256);
        ps_launch_mq(t, W, t->Q_pw, grad, mem, eta, k_or_rank, Q, ppart, status, pd, t->pd_pw, qd,
                     lazy_rank, st);
        int32_t* tdone = at<int32_t>(ws, lay.tdone);
        GCE_LAUNCH(ps_orth_kernel, wave_grid(int64_t(t->nps) * W, 8, r_orth), kPsOrthThreads, 0, st, t->d_layers, ps,
                   t->d_ps_layers, t->nps, W, 1, t->P_pw, t->ppart_pw, t->pd_pw, k_or_rank, ppart,
                   pd, P, status, t->ps_ntall, tdone, t->L, lazy_rank);
        if (t->ps_ntall > 0) {
            for (const PsOrthOp& op : ps_orth_ops(t->ps_tall_cap))
                GCE_LAUNCH(ps_orth_tall_kernel, wave_grid(int64_t(t->ps_tall_nunits) * W, 8, r_tall), 256, 0,
                           st, op, t->d_layers, ps, t->d_ps_tall_units, t->ps_tall_nunits, W, 1,
                           t->P_pw, t->ppart_pw, t->pd_pw, t->ps_ntall, t->ps_tall_parts,
                           k_or_rank, ppart, pd, at<double>(ws, lay.tparts),
                           at<double>(ws, lay.tscal), tdone, P);
        }
        ps_launch_mtp(t, W, t->pd_pw, mem, k_or_rank, pd, qpart, st);
        GCE_LAUNCH(ps_qred_kernel<false>, wave_grid(int64_t(t->psq_ntiles) * W, 8, r_qred), 256, 0,
                   st, t->d_layers, ps, t->d_psq_tiles, t->psq_ntiles, W, t->Q_pw, t->qpart_pw,
                   k_or_rank, qpart, Q, qd, nullptr, 1.0f);
        // the lazy step leaves M in the memory: the next step (or
        // gce_materialize_memory) takes P Q^T off
        if (!lazy_rank)
            ps_launch_resid(t, W, t->P_pw, t->Q_pw, t->pd_pw, k_or_rank, P, Q, pd, qd, mem,
                            dense_out, nullptr, st);
        if (check_launch() != GCE_OK) return GCE_ERR_CUDA;
    }
    return launch_dense_layers(t, W, grad, mem, eta, vals, status, st);
}

extern "C" int powersgd_step(const gce_table* t, int32_t W, const float* grad, float* mem, float eta,
                             const int32_t* k_or_rank, float* P, float* Q, float* vals,
                             float* dense_out, void* ws, size_t ws_bytes, void* stream) {
    return ps_step(t, W, grad, mem, eta, k_or_rank, P, Q, vals, dense_out, nullptr, ws, ws_bytes,
                   stream);
}

extern "C" int powersgd_step_lazy(const gce_table* t, int32_t W, const float* grad, float* mem,
                                  float eta, const int32_t* k_or_rank, float* P, float* Q,
                                  float* vals, int32_t* lazy_rank, void* ws, size_t ws_bytes,
                                  void* stream) {
    if (!lazy_rank || (reinterpret_cast<uintptr_t>(lazy_rank) & 3)) return GCE_ERR_ARG;
    return ps_step(t, W, grad, mem, eta, k_or_rank, P, Q, vals, nullptr, lazy_rank, ws, ws_bytes,
                   stream);
}

extern "C" int gce_materialize_memory(const gce_table* t, int32_t W, float* mem,
                                      int32_t* lazy_rank, void* ws, size_t ws_bytes,
                                      void* stream) {
    if (!t || W < 1 || !mem || !lazy_rank || !ws || !aligned16(mem) || !aligned16(ws))
        return GCE_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(lazy_rank) & 3) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_POWERSGD && t->ckind != -1) return GCE_ERR_KIND;
    const PsWs lay = ps_layout(t, W);
    if (ws_bytes < lay.total) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (t->nps > 0) {
        ps_launch_resid(t, W, t->P_pw, t->Q_pw, t->pd_pw, nullptr, nullptr, nullptr,
                        at<double>(ws, lay.pd), at<double>(ws, lay.qd), mem, nullptr, lazy_rank,
                        st);
        if (check_launch() != GCE_OK) return GCE_ERR_CUDA;
    }
    if (cudaMemsetAsync(lazy_rank, 0, sizeof(int32_t) * size_t(W) * size_t(t->L), st) !=
        cudaSuccess) {
        cudaGetLastError();
        return GCE_ERR_CUDA;
    }
    return GCE_OK;
}

extern "C" int powersgd_dp_step(const gce_table* t, int32_t W, const float* grad, float* mem,
                                float eta, const int32_t* k_or_rank, float* P, float* Q,
                                float* vals, void* ws, size_t ws_bytes, void* stream) {
    if (!t || W < 1 || !grad || !mem || !ws) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_POWERSGD && t->ckind != -1) return GCE_ERR_KIND;
    if (!aligned16(grad) || !aligned16(mem) || !aligned16(ws)) return GCE_ERR_ARG;
    if (t->nps > 0 && (!P || !Q || !aligned16(P) || !aligned16(Q))) return GCE_ERR_ARG;
    if (t->dtiles_pw > 0 && !vals) return GCE_ERR_ARG;
    if (k_or_rank && (reinterpret_cast<uintptr_t>(k_or_rank) & 3)) return GCE_ERR_ARG;
    const PsWs lay = ps_dp_layout(t, W);
    if (ws_bytes < lay.total) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = static_cast<int32_t*>(ws);
    const float inv_w = 1.0f / float(W);
    if (t->nps > 0) {
        double* ppart = at<double>(ws, lay.ppart);
        double* pd = at<double>(ws, lay.pd);
        double* qpart = at<double>(ws, lay.qpart);
        double* qd = at<double>(ws, lay.qd);
        float* qloc = at<float>(ws, lay.qloc);
        int32_t* tdone = at<int32_t>(ws, lay.tdone);
        const PsLayer* ps = static_cast<const PsLayer*>(t->d_ps);
        static const int r_orth = resident_blocks(ps_orth_kernel, kPsOrthThreads);
        static const int r_tall = resident_blocks(ps_orth_tall_kernel, 256);
        static const int r_qred = resident_blocks(ps_qred_kernel<true>, 256);
        // every worker reads the shared warm start Q (stride 0)
        ps_launch_mq(t, W, int64_t(0), grad, mem, eta, k_or_rank, Q, ppart, status, nullptr,
                     int64_t(0), nullptr, nullptr, st);
        // one P per layer from the partials of all W workers
        GCE_LAUNCH(ps_orth_kernel, wave_grid(t->nps, 8, r_orth), kPsOrthThreads, 0, st, t->d_layers, ps,
                   t->d_ps_layers, t->nps, 1, W, int64_t(0), t->ppart_pw, t->pd_pw, k_or_rank,
                   ppart, pd, P, status, t->ps_ntall, tdone, t->L, nullptr);
        if (t->ps_ntall > 0) {
            for (const PsOrthOp& op : ps_orth_ops(t->ps_tall_cap))
                GCE_LAUNCH(ps_orth_tall_kernel, wave_grid(t->ps_tall_nunits, 8, r_tall), 256, 0,
                           st, op, t->d_layers, ps, t->d_ps_tall_units, t->ps_tall_nunits, 1, W,
                           int64_t(0), t->ppart_pw, t->pd_pw, t->ps_ntall, t->ps_tall_parts,
                           k_or_rank, ppart, pd, at<double>(ws, lay.tparts),
                           at<double>(ws, lay.tscal), tdone, P);
        }
        // Q_w = M_w^T P for every worker with the shared P (stride 0)
        ps_launch_mtp(t, W, int64_t(0), mem, k_or_rank, pd, qpart, st);
        GCE_LAUNCH(ps_qred_kernel<true>, wave_grid(t->psq_ntiles, 8, r_qred), 256, 0, st,
                   t->d_layers, ps, t->d_psq_tiles, t->psq_ntiles, W, t->Q_pw, t->qpart_pw,
                   k_or_rank, qpart, qloc, qd, Q, inv_w);
        // each worker's error against its own Q_w (the shared fp64 P, stride 0)
        ps_launch_resid(t, W, int64_t(0), t->Q_pw, int64_t(0), k_or_rank, P, qloc, pd, qd, mem,
                        nullptr, nullptr, st);
        if (check_launch() != GCE_OK) return GCE_ERR_CUDA;
    }
    if (t->dtiles_pw > 0) {
        static const int r_dm = resident_blocks(ps_dense_mean_kernel, 256);
        GCE_LAUNCH(ps_dense_mean_kernel, wave_grid(t->dtiles_pw, 8, r_dm), 256, 0, st,
                   t->d_layers, t->d_dtile_layer, t->d_dtile_start, t->dtiles_pw, W, t->N, grad,
                   mem, eta, inv_w, vals, status);
        if (check_launch() != GCE_OK) return GCE_ERR_CUDA;
    }
    return GCE_OK;
}

// ---- data-parallel PowerSGD between ranks: the step cut at its two sums ------------------
static int ps_dp_check(const gce_table* t, const int32_t* k_or_rank, void* ws) {
    if (!t || !ws || !aligned16(ws)) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_POWERSGD && t->ckind != -1) return GCE_ERR_KIND;
    if (k_or_rank && (reinterpret_cast<uintptr_t>(k_or_rank) & 3)) return GCE_ERR_ARG;
    return GCE_OK;
}

extern "C" int gce_powersgd_dp_partials(const gce_table* t, int64_t* doubles_per_worker) {
    if (!t || !doubles_per_worker) return GCE_ERR_ARG;
    *doubles_per_worker = t->ppart_pw;
    return GCE_OK;
}

extern "C" int powersgd_dp_encode(const gce_table* t, int32_t W, const float* grad, float* mem,
                                  float eta, const int32_t* k_or_rank, const float* Q,
                                  double* Ppart, float* vals, void* ws, size_t ws_bytes,
                                  void* stream) {
    int rc = ps_dp_check(t, k_or_rank, ws);
    if (rc != GCE_OK) return rc;
    if (W < 1 || !grad || !mem || !aligned16(grad) || !aligned16(mem)) return GCE_ERR_ARG;
    if (t->nps > 0 && (!Q || !Ppart || !aligned16(Q) || !aligned16(Ppart))) return GCE_ERR_ARG;
    if (t->dtiles_pw > 0 && (!vals || !aligned16(vals))) return GCE_ERR_ARG;
    if (ws_bytes < ps_dp_layout(t, W).total) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = static_cast<int32_t*>(ws);
    if (t->nps > 0) {
        // every worker reads the shared warm start Q (stride 0)
        ps_launch_mq(t, W, int64_t(0), grad, mem, eta, k_or_rank, Q, Ppart, status, nullptr,
                     int64_t(0), nullptr, nullptr, st);
        if (check_launch() != GCE_OK) return GCE_ERR_CUDA;
    }
    // DENSE layers: each worker's residual as its payload row, memory -> 0
    return launch_dense_layers(t, W, grad, mem, eta, vals, status, st);
}

extern "C" int powersgd_dp_orthogonalize(const gce_table* t, int32_t W, const int32_t* k_or_rank,
                                         const double* Ppart, float* P, void* ws, size_t ws_bytes,
                                         void* stream) {
    int rc = ps_dp_check(t, k_or_rank, ws);
    if (rc != GCE_OK) return rc;
    if (W < 1) return GCE_ERR_ARG;
    if (t->nps == 0) return GCE_OK;
    if (!Ppart || !P || !aligned16(Ppart) || !aligned16(P)) return GCE_ERR_ARG;
    // the W-independent head of the workspace (any W it was sized for)
    const PsWs lay = ps_dp_layout(t, 1);
    if (ws_bytes < lay.ppart) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = static_cast<int32_t*>(ws);
    const PsLayer* ps = static_cast<const PsLayer*>(t->d_ps);
    double* pd = at<double>(ws, lay.pd);
    int32_t* tdone = at<int32_t>(ws, lay.tdone);
    static const int r_orth = resident_blocks(ps_orth_kernel, kPsOrthThreads);
    static const int r_tall = resident_blocks(ps_orth_tall_kernel, 256);
    // one P per layer from the partials of all W workers, in worker order
    GCE_LAUNCH(ps_orth_kernel, wave_grid(t->nps, 8, r_orth), kPsOrthThreads, 0, st, t->d_layers, ps,
               t->d_ps_layers, t->nps, 1, W, int64_t(0), t->ppart_pw, t->pd_pw, k_or_rank, Ppart,
               pd, P, status, t->ps_ntall, tdone, t->L, nullptr);
    if (t->ps_ntall > 0) {
        for (const PsOrthOp& op : ps_orth_ops(t->ps_tall_cap))
            GCE_LAUNCH(ps_orth_tall_kernel, wave_grid(t->ps_tall_nunits, 8, r_tall), 256, 0, st,
                       op, t->d_layers, ps, t->d_ps_tall_units, t->ps_tall_nunits, 1, W,
                       int64_t(0), t->ppart_pw, t->pd_pw, t->ps_ntall, t->ps_tall_parts,
                       k_or_rank, Ppart, pd, at<double>(ws, lay.tparts),
                       at<double>(ws, lay.tscal), tdone, P);
    }
    return check_launch();
}

extern "C" int powersgd_dp_project(const gce_table* t, int32_t W, float* mem,
                                   const int32_t* k_or_rank, float* Qw, void* ws,
                                   size_t ws_bytes, void* stream) {
    int rc = ps_dp_check(t, k_or_rank, ws);
    if (rc != GCE_OK) return rc;
    if (W < 1 || !mem || !aligned16(mem)) return GCE_ERR_ARG;
    if (t->nps == 0) return GCE_OK;
    if (!Qw || !aligned16(Qw)) return GCE_ERR_ARG;
    const PsWs lay = ps_dp_layout(t, W);
    if (ws_bytes < lay.total) return GCE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const PsLayer* ps = static_cast<const PsLayer*>(t->d_ps);
    double* pd = at<double>(ws, lay.pd);
    double* qpart = at<double>(ws, lay.qpart);
    double* qd = at<double>(ws, lay.qd);
    static const int r_qred = resident_blocks(ps_qred_kernel<false>, 256);
    // Q_w = M_w^T P for this rank's workers with the shared P (stride 0)
    ps_launch_mtp(t, W, int64_t(0), mem, k_or_rank, pd, qpart, st);
    GCE_LAUNCH(ps_qred_kernel<false>, wave_grid(int64_t(t->psq_ntiles) * W, 8, r_qred), 256, 0,
               st, t->d_layers, ps, t->d_psq_tiles, t->psq_ntiles, W, t->Q_pw, t->qpart_pw,
               k_or_rank, qpart, Qw, qd, nullptr, 1.0f);
    // each worker's error against its own Q_w
    ps_launch_resid(t, W, int64_t(0), t->Q_pw, int64_t(0), k_or_rank, nullptr, nullptr, pd, qd,
                    mem, nullptr, nullptr, st);
    return check_launch();
}

extern "C" int powersgd_dp_mean(const gce_table* t, int32_t W, const int32_t* k_or_rank,
                                const float* Qw, float* Q, const float* vals_all, float* vals,
                                void* stream) {
    if (!t || W < 1) return GCE_ERR_ARG;
    if (t->ckind != GCE_KIND_POWERSGD && t->ckind != -1) return GCE_ERR_KIND;
    if (k_or_rank && (reinterpret_cast<uintptr_t>(k_or_rank) & 3)) return GCE_ERR_ARG;
    if (t->nps > 0 && (!Qw || !Q)) return GCE_ERR_ARG;
    if (t->dtiles_pw > 0 && (!vals_all || !vals)) return GCE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const float inv_w = 1.0f / float(W);
    if (t->nps > 0) {
        static const int r_qm = resident_blocks(ps_qmean_kernel, 256);
        GCE_LAUNCH(ps_qmean_kernel, wave_grid(t->psq_ntiles, 8, r_qm), 256, 0, st, t->d_layers,
                   t->d_psq_tiles, t->psq_ntiles, W, t->Q_pw, k_or_rank, Qw, Q, inv_w);
    }
    if (t->dtiles_pw > 0) {
        static const int r_vm = resident_blocks(ps_vmean_kernel, 256);
        GCE_LAUNCH(ps_vmean_kernel, wave_grid(t->dtiles_pw, 8, r_vm), 256, 0, st, t->d_layers,
                   t->d_dtile_layer, t->d_dtile_start, t->dtiles_pw, W, t->vals_pw, vals_all, vals,
                   inv_w);
    }
    return check_launch();
}
