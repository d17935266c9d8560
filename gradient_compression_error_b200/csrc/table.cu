// table.cu -- layer table, workspace queries, status word, launch counter,
// and the kernel for uncompressed (DENSE) layers shared by every step.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "topk_layout.cuh"

namespace gce {

std::atomic<uint64_t> g_launches{0};
std::atomic<bool> g_prof_on{false};

bool programmatic_launch() {
    static const bool on = [] {
        const char* v = std::getenv("GCE_PROGRAMMATIC_LAUNCH");
        return !(v && v[0] == '0');
    }();
    return on;
}

// ---- launch timing (host side) -------------------------------------------------
namespace {
struct ProfRec {
    const char* name;
    cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_pool;
size_t g_prof_used = 0;
constexpr size_t kProfMax = 1 << 16;
struct ProfAgg {
    std::string name;
    double ms;
    int64_t n;
};
std::vector<ProfAgg> g_prof_agg;
std::string g_prof_only;  // record only kernels whose name starts with this (empty: all)

cudaEvent_t prof_event() {
    if (g_prof_used < g_prof_pool.size()) return g_prof_pool[g_prof_used++];
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    g_prof_pool.push_back(e);
    ++g_prof_used;
    return e;
}
}  // namespace

void prof_before(const char* name, cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (g_prof_recs.size() >= kProfMax) return;
    if (!g_prof_only.empty() && std::strncmp(name, g_prof_only.c_str(), g_prof_only.size()) != 0)
        return;
    ProfRec r{name, prof_event(), nullptr};
    if (!r.a) return;
    cudaEventRecord(r.a, st);
    g_prof_recs.push_back(r);
}

void prof_after(cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (g_prof_recs.empty() || g_prof_recs.back().b) return;
    ProfRec& r = g_prof_recs.back();
    r.b = prof_event();
    if (r.b) cudaEventRecord(r.b, st);
}

// ---- settings: process-wide values and each table's own -------------------------
namespace {
// defaults: bracket margin 6 sigma, rand-k look-ahead on, signSGD look-ahead
// from L2 (-1), wait test off
std::atomic<double> g_opt[4] = {6.0, 1.0, -1.0, 0.0};

bool option_valid(int opt, double v) {
    switch (opt) {
        case GCE_OPT_BRACKET_SIGMA: return v > -100.0 && v < 100.0;
        case GCE_OPT_RANDK_AHEAD:
        case GCE_OPT_SIGN_EMIT_FIRST: return v == 0.0 || v == 1.0;
        case GCE_OPT_SIGN_AHEAD:
            return v >= -1.0 && v <= double(1 << 20) && v == std::floor(v);
        default: return false;
    }
}

int set_process_option(int opt, double v) {
    if (!option_valid(opt, v)) return GCE_ERR_ARG;
    g_opt[opt].store(v);
    return GCE_OK;
}
}  // namespace

double option_of(const gce_table* t, int opt) {
    const double v = t ? t->opt[opt].load(std::memory_order_relaxed) : NAN;
    return std::isnan(v) ? g_opt[opt].load(std::memory_order_relaxed) : v;
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// ---- DENSE layers: payload = fl32(m + fl32(eta*g)), memory -> +0 ----------

__global__ void __launch_bounds__(256) dense_kernel(const DevLayer* __restrict__ layers,
                                                    const int32_t* __restrict__ dtile_layer,
                                                    const int32_t* __restrict__ dtile_start,
                                                    int32_t dtiles_pw, int32_t W, int64_t N,
                                                    int64_t vals_pw, const float* __restrict__ grad,
                                                    float* __restrict__ mem, float eta,
                                                    float* __restrict__ vals,
                                                    int32_t* __restrict__ status) {
    grid_dependency_sync();
    const int64_t total = int64_t(dtiles_pw) * W;
    bool bad = false;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
        const int w = int(t / dtiles_pw);
        const int lt = int(t % dtiles_pw);
        const DevLayer L = layers[dtile_layer[lt]];
        const int64_t start = dtile_start[lt];
        const int64_t cnt = min64(kDenseTile, L.n - start);
        const float* g = grad + int64_t(w) * N + L.offset + start;
        float* m = mem + int64_t(w) * N + L.offset + start;
        float* out = vals + int64_t(w) * vals_pw + L.val_off + start;
        for (int64_t i = threadIdx.x; i < cnt; i += blockDim.x) {
            const float v = residual(m[i], eta, __ldcs(g + i));
            bad |= abs_key(v) >= kNonFiniteKey;
            out[i] = v;
            m[i] = 0.0f;
        }
    }
    flag_nonfinite(bad, status);
}

int launch_dense_layers(const gce_table* t, int32_t W, const float* grad, float* mem, float eta,
                        float* vals, int32_t* status, cudaStream_t st) {
    if (t->dtiles_pw == 0) return GCE_OK;
    if (!vals) return GCE_ERR_ARG;
    int64_t total = int64_t(t->dtiles_pw) * W;
    static const int r_dense = resident_blocks(dense_kernel, 256);
    const int grid = wave_grid(total, 8, r_dense);
    GCE_LAUNCH(dense_kernel, grid, 256, 0, st, t->d_layers, t->d_dtile_layer, t->d_dtile_start,
               t->dtiles_pw, W, t->N, t->vals_pw, grad, mem, eta, vals, status);
    return check_launch();
}

}  // namespace gce

using namespace gce;

static void free_table(gce_table* t) {
    if (!t) return;
    cudaFree(t->d_layers);
    cudaFree(t->d_comp);
    cudaFree(t->d_dense);
    cudaFree(t->d_tile_layer);
    cudaFree(t->d_tile_info);
    cudaFree(t->d_sunit_layer);
    cudaFree(t->d_sunit_part);
    cudaFree(t->d_dtile_layer);
    cudaFree(t->d_dtile_start);
    cudaFree(t->d_dc_tile_layer);
    cudaFree(t->d_dc_nl_tiles);
    cudaFree(t->d_dc_sp_info);
    cudaFree(t->d_dc_dn_tiles);
    cudaFree(t->d_bunit_layer);
    cudaFree(t->d_bunit_chunk);
    powersgd_plan_free(t);
    accordion_plan_free(t);
    sign_plan_free(t);
    delete t;
}

template <class T>
static int upload(T** dst, const std::vector<T>& src) {
    *dst = nullptr;
    if (src.empty()) return GCE_OK;
    if (cudaMalloc(dst, src.size() * sizeof(T)) != cudaSuccess) return GCE_ERR_NOMEM;
    if (cudaMemcpy(*dst, src.data(), src.size() * sizeof(T), cudaMemcpyHostToDevice) != cudaSuccess)
        return GCE_ERR_CUDA;
    return GCE_OK;
}

extern "C" int gce_table_create(const gce_layer_desc* descs, int32_t L, gce_table** out) {
    if (!descs || !out || L < 1) return GCE_ERR_ARG;
    *out = nullptr;
    gce_table* t = new gce_table();
    t->L = L;
    int64_t off = 0, voff = 0, poff = 0, qoff = 0, spoff = 0;
    int32_t tiles = 0;
    std::vector<int32_t> tile_layer, sunit_layer, sunit_part, dtile_layer, dtile_start;
    std::vector<TileInfo> tile_info;
    std::vector<int32_t> dc_tile_layer, bunit_layer, bunit_chunk, dc_nl, dc_dn;
    std::vector<DcTileInfo> dc_sp;
    int32_t dc_tiles = 0, dc_slots = 0;
    for (int32_t l = 0; l < L; ++l) {
        const gce_layer_desc& d = descs[l];
        const int64_t n = d.rows * d.cols;
        if (d.rows < 1 || d.cols < 1 || n > INT32_MAX || d.kind < 0 || d.kind > GCE_KIND_SIGN) {
            delete t;
            return GCE_ERR_ARG;
        }
        DevLayer x{};
        x.offset = off;
        x.n = n;
        x.rows = d.rows;
        x.cols = d.cols;
        x.kind = d.kind;
        x.cap = d.cap;
        x.val_off = x.p_off = x.q_off = -1;
        x.sp_off = -1;
        x.sidx = -1;
        if (d.kind == GCE_KIND_TOPK || d.kind == GCE_KIND_RANDK) {
            if (d.cap < 1 || d.cap > n) { delete t; return GCE_ERR_ARG; }
            x.val_off = voff;
            voff += (d.cap + 3) & ~int64_t(3);  // keep every slice 16-byte aligned
        } else if (d.kind == GCE_KIND_POWERSGD) {
            if (d.cap < 1 || d.cap > kMaxRank || d.cap > d.rows || d.cap > d.cols) {
                delete t;
                return GCE_ERR_ARG;
            }
            x.p_off = poff;
            x.q_off = qoff;
            poff += (d.rows * d.cap + 3) & ~int64_t(3);
            qoff += (d.cols * d.cap + 3) & ~int64_t(3);
        } else if (d.kind == GCE_KIND_SIGN) {
            // slot 0: the scale, slots 1-3: zero, then the sign words
            x.val_off = voff;
            voff += 4 + ((((n + 31) / 32) + 3) & ~int64_t(3));
        } else {  // DENSE
            x.val_off = voff;
            voff += (n + 3) & ~int64_t(3);
            for (int64_t s = 0; s < n; s += kDenseTile) {
                dtile_layer.push_back(l);
                dtile_start.push_back(int32_t(s));
            }
            t->dense.push_back(l);
            t->dense_N += n;
        }
        if (d.kind != GCE_KIND_DENSE) {
            if (t->ckind >= 0 && t->ckind != d.kind) { delete t; return GCE_ERR_KIND; }
            t->ckind = d.kind;
            x.sidx = int32_t(t->comp.size());
            x.sp_off = spoff;
            spoff += n;
            t->comp.push_back(l);
            t->max_comp_n = std::max(t->max_comp_n, n);
            if (d.kind != GCE_KIND_POWERSGD) {
                x.tile0 = tiles;
                x.ntiles = int32_t((n + kTkTile - 1) / kTkTile);
                for (int32_t i = 0; i < x.ntiles; ++i) {
                    tile_layer.push_back(l);
                    tile_info.push_back(TileInfo{x.offset, x.sp_off, x.val_off, x.sidx,
                                                 int32_t(int64_t(i) * kTkTile)});
                }
                tiles += x.ntiles;
                const int32_t parts = int32_t((n + kTkSamplePart - 1) / kTkSamplePart);
                for (int32_t p = 0; p < parts; ++p) {
                    sunit_layer.push_back(l);
                    sunit_part.push_back(p);
                }
            }
        }
        x.dc_tile0 = dc_tiles;
        x.dc_ntiles = int32_t((n + kDcTile - 1) / kDcTile);
        x.dc_base = dc_slots;
        for (int32_t i = 0; i < x.dc_ntiles; ++i) {
            if (d.kind != GCE_KIND_POWERSGD) dc_nl.push_back(dc_tiles + i);
            if (d.kind == GCE_KIND_TOPK || d.kind == GCE_KIND_RANDK) {
                DcTileInfo r{};
                r.tstart = int32_t(int64_t(i) * kDcTile);
                r.out_off = x.offset + r.tstart;
                r.val_off = x.val_off;
                r.cnt = int32_t(std::min<int64_t>(kDcTile, n - r.tstart));
                r.bslot = dc_slots + int32_t((int64_t(i) * kDcTile) >> kDcSpanLog);
                r.layer = l;
                r.cap = d.cap;
                dc_sp.push_back(r);
            }
            if (d.kind == GCE_KIND_DENSE) dc_dn.push_back(dc_tiles + i);
            dc_tile_layer.push_back(l);
        }
        dc_tiles += x.dc_ntiles;
        dc_slots += int32_t((n + kDcSpan - 1) / kDcSpan) + 1;
        if (d.kind == GCE_KIND_TOPK || d.kind == GCE_KIND_RANDK) {
            const int32_t chunks = (d.cap + kDcBoundChunk - 1) / kDcBoundChunk;
            for (int32_t c = 0; c < chunks; ++c) {
                bunit_layer.push_back(l);
                bunit_chunk.push_back(c);
            }
        }
        off += n;
        t->layers.push_back(x);
    }
    t->N = off;
    t->vals_pw = voff;
    t->P_pw = poff;
    t->Q_pw = qoff;
    t->comp_N = spoff;
    t->tiles_pw = tiles;
    t->sunits_pw = int32_t(sunit_layer.size());
    t->dtiles_pw = int32_t(dtile_layer.size());
    t->dc_tiles = dc_tiles;
    t->dc_slots = dc_slots;
    t->bunits_pw = int32_t(bunit_layer.size());
    int rc = GCE_OK;
    if (rc == GCE_OK) rc = upload(&t->d_layers, t->layers);
    if (rc == GCE_OK) rc = upload(&t->d_comp, t->comp);
    if (rc == GCE_OK) rc = upload(&t->d_dense, t->dense);
    if (rc == GCE_OK) rc = upload(&t->d_tile_layer, tile_layer);
    if (rc == GCE_OK) rc = upload(&t->d_tile_info, tile_info);
    if (rc == GCE_OK) rc = upload(&t->d_sunit_layer, sunit_layer);
    if (rc == GCE_OK) rc = upload(&t->d_sunit_part, sunit_part);
    if (rc == GCE_OK) rc = upload(&t->d_dtile_layer, dtile_layer);
    if (rc == GCE_OK) rc = upload(&t->d_dtile_start, dtile_start);
    if (rc == GCE_OK) rc = upload(&t->d_dc_tile_layer, dc_tile_layer);
    t->dc_nl_n = int32_t(dc_nl.size());
    if (rc == GCE_OK) rc = upload(&t->d_dc_nl_tiles, dc_nl);
    t->dc_sp_n = int32_t(dc_sp.size());
    if (rc == GCE_OK) rc = upload(&t->d_dc_sp_info, dc_sp);
    t->dc_dn_n = int32_t(dc_dn.size());
    if (rc == GCE_OK) rc = upload(&t->d_dc_dn_tiles, dc_dn);
    if (rc == GCE_OK) rc = upload(&t->d_bunit_layer, bunit_layer);
    if (rc == GCE_OK) rc = upload(&t->d_bunit_chunk, bunit_chunk);
    if (rc == GCE_OK) rc = powersgd_plan(t);
    if (rc == GCE_OK) rc = accordion_plan(t);
    if (rc != GCE_OK) {
        free_table(t);
        return rc;
    }
    *out = t;
    return GCE_OK;
}

extern "C" int gce_table_destroy(gce_table* t) {
    if (!t) return GCE_ERR_ARG;
    free_table(t);
    return GCE_OK;
}

extern "C" int gce_table_get_totals(const gce_table* t, gce_table_totals* out) {
    if (!t || !out) return GCE_ERR_ARG;
    out->L = t->L;
    out->N = t->N;
    out->vals_per_worker = t->vals_pw;
    out->P_per_worker = t->P_pw;
    out->Q_per_worker = t->Q_pw;
    out->compressed_kind = t->ckind;
    return GCE_OK;
}

extern "C" int gce_table_get_layer(const gce_table* t, int32_t l, gce_layer_info* out) {
    if (!t || !out || l < 0 || l >= t->L) return GCE_ERR_ARG;
    const DevLayer& x = t->layers[l];
    out->offset = x.offset;
    out->n = x.n;
    out->rows = x.rows;
    out->cols = x.cols;
    out->kind = x.kind;
    out->cap = x.cap;
    out->val_offset = x.val_off;
    out->p_offset = x.p_off;
    out->q_offset = x.q_off;
    return GCE_OK;
}

namespace gce {
size_t topk_ws_bytes(const gce_table* t, int32_t W);
size_t randk_ws_bytes(const gce_table* t, int32_t W);
size_t powersgd_ws_bytes(const gce_table* t, int32_t W);
size_t powersgd_dp_ws_bytes(const gce_table* t, int32_t W);
size_t sign_ws_bytes(const gce_table* t, int32_t W);
size_t accordion_ws_bytes(const gce_table* t);
size_t decompress_ws_bytes(const gce_table* t, int32_t W);
}  // namespace gce

extern "C" int gce_workspace_bytes(const gce_table* t, int32_t W, int32_t op, size_t* bytes) {
    if (!t || !bytes || W < 1) return GCE_ERR_ARG;
    switch (op) {
        case GCE_OP_TOPK: *bytes = topk_ws_bytes(t, W); break;
        case GCE_OP_RANDK: *bytes = randk_ws_bytes(t, W); break;
        case GCE_OP_POWERSGD: *bytes = powersgd_ws_bytes(t, W); break;
        case GCE_OP_ACCORDION: *bytes = accordion_ws_bytes(t); break;
        case GCE_OP_DECOMPRESS: *bytes = decompress_ws_bytes(t, W); break;
        case GCE_OP_POWERSGD_DP: *bytes = powersgd_dp_ws_bytes(t, W); break;
        case GCE_OP_SIGN: *bytes = sign_ws_bytes(t, W); break;
        default: return GCE_ERR_ARG;
    }
    return GCE_OK;
}

extern "C" int gce_status(void* ws, void* stream, int32_t* status) {
    if (!ws || !status) return GCE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, ws, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return GCE_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof h, st) != cudaSuccess) return GCE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GCE_ERR_CUDA;
    *status = h;
    return GCE_OK;
}

extern "C" uint64_t gce_launch_count(void) { return g_launches.load(); }

extern "C" int gce_profile_start(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_recs.clear();
    g_prof_agg.clear();
    g_prof_used = 0;
    g_prof_on.store(true);
    return GCE_OK;
}

extern "C" int gce_profile_only(const char* name_prefix) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_only = name_prefix ? name_prefix : "";
    return GCE_OK;
}

extern "C" int gce_profile_stop(void) {
    g_prof_on.store(false);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    int rc = GCE_OK;
    for (const ProfRec& r : g_prof_recs) {
        if (!r.a || !r.b) continue;
        if (cudaEventSynchronize(r.b) != cudaSuccess) { rc = GCE_ERR_CUDA; continue; }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) { rc = GCE_ERR_CUDA; continue; }
        bool found = false;
        for (ProfAgg& a : g_prof_agg)
            if (a.name == r.name) {
                a.ms += ms;
                a.n += 1;
                found = true;
                break;
            }
        if (!found) g_prof_agg.push_back(ProfAgg{r.name, double(ms), 1});
    }
    g_prof_recs.clear();
    return rc;
}

extern "C" int gce_profile_count(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    return int(g_prof_agg.size());
}

extern "C" int gce_profile_get(int32_t i, char* name, int32_t name_len, double* total_ms,
                               int64_t* launches) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (i < 0 || size_t(i) >= g_prof_agg.size() || !name || name_len < 1 || !total_ms || !launches)
        return GCE_ERR_ARG;
    const ProfAgg& a = g_prof_agg[i];
    std::strncpy(name, a.name.c_str(), size_t(name_len) - 1);
    name[name_len - 1] = 0;
    *total_ms = a.ms;
    *launches = a.n;
    return GCE_OK;
}

extern "C" const char* gce_error_string(int code) {
    switch (code) {
        case GCE_OK: return "ok";
        case GCE_ERR_ARG: return "invalid argument";
        case GCE_ERR_CUDA: return "CUDA runtime error";
        case GCE_ERR_WORKSPACE: return "workspace missing or too small";
        case GCE_ERR_NOMEM: return "device allocation failed";
        case GCE_ERR_KIND: return "layer kinds do not fit this call";
        default: return "unknown error";
    }
}

extern "C" int gce_set_bracket_sigma(double sigma) {
    return set_process_option(GCE_OPT_BRACKET_SIGMA, sigma);
}

extern "C" int gce_set_randk_ahead(int32_t on) {
    return set_process_option(GCE_OPT_RANDK_AHEAD, double(on));
}

extern "C" int gce_set_sign_ahead(int32_t tiles) {
    return set_process_option(GCE_OPT_SIGN_AHEAD, double(tiles));
}

extern "C" int gce_set_sign_emit_first(int32_t on) {
    return set_process_option(GCE_OPT_SIGN_EMIT_FIRST, double(on));
}

extern "C" int gce_table_set_option(gce_table* t, int32_t option, double value) {
    if (!t || option < 0 || option > 3 || !option_valid(option, value)) return GCE_ERR_ARG;
    t->opt[option].store(value);
    return GCE_OK;
}

extern "C" int gce_table_reset_option(gce_table* t, int32_t option) {
    if (!t || option < 0 || option > 3) return GCE_ERR_ARG;
    t->opt[option].store(NAN);
    return GCE_OK;
}

extern "C" int gce_table_get_option(const gce_table* t, int32_t option, double* value) {
    if (!t || option < 0 || option > 3 || !value) return GCE_ERR_ARG;
    *value = option_of(t, option);
    return GCE_OK;
}
