// wam_video_prefill_kv_fuse_noalloc: the video prefill with the Interval KV-Fusion epilogue
// for callers that cannot allocate device memory.
//
// The fusion epilogue needs an fp32 accumulator that lives across the calls of one interval.
// wam_video_prefill_kv takes it from the caller (acc_k, acc_v).  Some callers cannot call
// cudaMalloc: code running while a CUDA graph is being captured, plug-ins handed a fixed
// memory pool by their host, or embedded runtimes that allocate everything at start-up.  This
// entry point keeps the accumulator in a file-scope device array instead, so the caller passes
// only its inputs and outputs.  It runs exactly the same kernels as wam_video_prefill_kv.
#include <cstdio>

#include "launch.h"

// The accumulator: K half then V half, WAM_NOALLOC_FUSE_ACC_ELEMS floats each (2 x 16 MiB).
// Every GPU that loads this code holds it until the process exits.  In host code the name is
// only a host-side stand-in: kernels receive the device address from cudaGetSymbolAddress.
static __device__ __align__(256) float g_noalloc_fuse_acc[2 * size_t(WAM_NOALLOC_FUSE_ACC_ELEMS)];

namespace {

// Device address of the accumulator on the current device.  It is looked up on every call
// (cudaGetSymbolAddress allocates nothing): an address kept from an earlier call could belong
// to a context that a device reset has since replaced.
float* noalloc_acc_address(wam_status* st) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_fuse_acc);
  if (e != cudaSuccess || !p) {
    char msg[256];
    snprintf(msg, sizeof(msg), "wam_video_prefill_kv_fuse_noalloc: cudaGetSymbolAddress: %s",
             cudaGetErrorString(e));
    *st = wam::record_error(WAM_ERR_CUDA, msg);
    return nullptr;
  }
  return static_cast<float*>(p);
}

}  // namespace

extern "C" wam_status wam_video_prefill_kv_fuse_noalloc(
    const wam_video_layout* layout, wam_dtype dt, int32_t f_begin, int32_t f_end, const void* q,
    const void* k_new, const void* v_new, void* k_cache, void* v_cache, int32_t store_kv, void* o,
    wam_dtype o_dt, float weight, int32_t first_in_interval, int32_t last_in_interval,
    void* fused_k, void* fused_v, wam_stream_t stream) {
  if (!layout)
    return wam::record_error(WAM_ERR_INVALID_ARGUMENT, "layout is NULL");
  if (layout->B < 1 || layout->F < 1 || layout->T < 1 || layout->H < 1 || layout->D < 1)
    return wam::record_error(WAM_ERR_INVALID_ARGUMENT, "B, F, T, H and D must be >= 1");
  // A one-layer interval (first and last) writes the fused pair directly and never touches
  // the accumulator, so only calls that do are held to the array's size.
  const bool uses_acc = !(first_in_interval && last_in_interval);
  const long long need = (long long)layout->B * layout->F * layout->T * layout->H * layout->D;
  if (uses_acc && need > (long long)WAM_NOALLOC_FUSE_ACC_ELEMS) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "wam_video_prefill_kv_fuse_noalloc: B*F*T*H*D = %lld exceeds the static accumulator "
             "of WAM_NOALLOC_FUSE_ACC_ELEMS = %lld elements; use wam_video_prefill_kv with a "
             "caller-owned accumulator",
             need, (long long)WAM_NOALLOC_FUSE_ACC_ELEMS);
    return wam::record_error(WAM_ERR_UNSUPPORTED, msg);
  }
  wam_status st = WAM_OK;
  float* acc = noalloc_acc_address(&st);
  if (!acc) return st;
  wam_fuse_epilogue e;
  e.weight = weight;
  e.first_in_interval = first_in_interval;
  e.last_in_interval = last_in_interval;
  e.acc_k = acc;
  e.acc_v = acc + size_t(WAM_NOALLOC_FUSE_ACC_ELEMS);
  e.fused_k = fused_k;
  e.fused_v = fused_v;
  return wam_video_prefill_kv(layout, dt, f_begin, f_end, q, k_new, v_new, k_cache, v_cache,
                              store_kv, o, o_dt, &e, stream);
}
