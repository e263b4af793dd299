// Internal launchers shared by the C-ABI layer (host code only).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace wam {

cudaError_t launch_euler(int64_t n, float* x, const float* v, float dsigma, cudaStream_t s);
cudaError_t launch_store_fuse(const PrefillArgs& a, int D, bool bf16, cudaStream_t s);
cudaError_t launch_fuse(const FuseArgs& a, int D, bool bf16, cudaStream_t s);
cudaError_t launch_copy_frames(const CopyArgs& a, cudaStream_t s);
cudaError_t launch_debug_mask(const PrefillArgs& a, uint8_t* mask, cudaStream_t s);
cudaError_t launch_prefill_simt(const PrefillArgs& a, int D, bool bf16, cudaStream_t s);
cudaError_t launch_action_simt(const ActionArgs& a, int D, bool bf16, cudaStream_t s);
cudaError_t launch_wait_timeout(uint32_t polls, int* err, cudaStream_t s);
cudaError_t launch_nvfp4_encode(Nvfp4Args& a, cudaStream_t s);

// Tensor-core paths (bf16, D = 128).  Return cudaErrorNotSupported when the shape has no
// tensor-core kernel; the caller then takes the CUDA-core path.
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s);   // tcgen05 + TMEM
cudaError_t launch_action_tc(const ActionArgs& a, cudaStream_t s);
cudaError_t launch_action_nvfp4(const ActionArgs& a, cudaStream_t s);  // T % 128 == 0, bf16 action inputs
int action_tc_total_tiles(const ActionArgs& a);
int action_tc_max_parts(const ActionArgs& a, int P, int G);
size_t action_tc_workspace_bytes(int BH, int max_parts);
// The aligned split of the 128-key reads (T % 128 == 0): sets kparts, G, P (the CTA count) and
// max_parts; returns P.
int action_aligned_plan(ActionArgs& a, int sms);
// The action-read workspace starts with a fixed ticket region, so tickets never land on
// partial data of an earlier call with another layout; partial slots follow it.
constexpr size_t kTicketBytes = 65536;  // one int per (episode, head): B * H <= 16384

// Tensor map of a token-major bf16 tensor [B, ntok, H, 128] with a box of 64 x rows
// (128B swizzle), rows along the token dimension.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int B, int ntok, int H, int box_rows);

// Sets the calling thread's wam_last_error() message and returns st.
wam_status record_error(wam_status st, const char* msg);

// Launch with programmatic stream serialization (and an optional 1-D cluster size > 0): the
// kernel's CTAs may be scheduled while the previous kernel on the stream drains; the kernel
// calls grid_dependency_wait() before it touches global memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster > 0) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace wam
