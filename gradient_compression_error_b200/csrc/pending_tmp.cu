// temporary: entry points not yet implemented (replaced by randk.cu, powersgd.cu, accordion.cu)
#include "common.cuh"
namespace gce {
size_t powersgd_ws_bytes(const gce_table*, int32_t) { return GCE_WS_HEADER_BYTES; }
size_t accordion_ws_bytes(const gce_table*) { return GCE_WS_HEADER_BYTES; }
}
extern "C" int powersgd_init_q(const gce_table*, int32_t, uint64_t, float*, void*) { return GCE_ERR_KIND; }
extern "C" int powersgd_step(const gce_table*, int32_t, const float*, float*, float, const int32_t*, float*, float*, float*, float*, void*, size_t, void*) { return GCE_ERR_KIND; }
extern "C" int accordion_init(const gce_table*, double*, int32_t*, void*) { return GCE_ERR_KIND; }
extern "C" int accordion_select(const gce_table*, const float*, int64_t, int32_t, double, int32_t, int32_t, double*, int32_t*, double*, int32_t*, void*, size_t, void*) { return GCE_ERR_KIND; }
