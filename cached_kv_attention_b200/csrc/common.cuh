// Shared definitions of the WAM attention kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wam.h"

namespace wam {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------------------
// Per-launch work tables (kernel parameters, built on the host from the padding mask and
// the attention blocks).  A frame of an episode is a contiguous run of T*H*D elements in
// every token-major tensor, so all work is addressed by (episode, frame).
// ---------------------------------------------------------------------------------------

// item = b | f << 10 | nk << 21: query frame f of episode b reads the first nk entries of
// that episode's valid-frame list (keys of blocks <= its own, padding frames left out).
__host__ __device__ inline uint32_t pack_item(int b, int f, int nk) {
  return uint32_t(b) | (uint32_t(f) << 10) | (uint32_t(nk) << 21);
}
__host__ __device__ inline int item_b(uint32_t it) { return int(it & 1023u); }
__host__ __device__ inline int item_f(uint32_t it) { return int((it >> 10) & 2047u); }
__host__ __device__ inline int item_nk(uint32_t it) { return int(it >> 21); }

struct FrameLists {
  int32_t n_items;                               // prefill / store: valid query frames
  int32_t paired;                                // tensor-core prefill: items (2i, 2i + 1) share CTAs
  uint32_t item[WAM_MAX_EPISODE_FRAMES];         // launch order (order_items_for_tc in api.cu)
  uint16_t vlist[WAM_MAX_EPISODE_FRAMES];        // valid frames of episode b at [b*F, ...)
  uint16_t nvalid[WAM_MAX_EPISODE_FRAMES];       // number of valid frames of episode b
};

struct PrefillArgs {
  const void* q;
  const void* k_new;
  const void* v_new;
  const void* k_cache;  // keys of frames < f_begin
  const void* v_cache;
  void* k_store;        // non-null: store new K/V of the call's valid frames
  void* v_store;
  void* o;
  float* acc_k;
  float* acc_v;
  void* fused_k;
  void* fused_v;
  float fuse_w;
  int32_t fuse_on, fuse_first, fuse_last;
  int32_t B, H, T, F, f_begin, f_end;
  int32_t o_f32;
  float scale_log2;  // softmax scale * log2(e)
  int* err;          // device error word (a bounded wait that gave up writes WAM_ERR_TIMEOUT)
  FrameLists fl;
};

struct ActionArgs {
  const void* fk;  // fused video K/V or null
  const void* fv;
  const void* qa;
  const void* ka;
  const void* va;
  void* o;
  int32_t B, H, T, F, n_act;
  int32_t o_f32;
  int32_t with_video;
  int32_t P;          // CTAs of the persistent grid
  int32_t G;          // tiles of the whole call (all episodes and heads)
  int32_t max_parts;  // workspace slots per (episode, head)
  // 128-key reads: every head of episode b is cut into kparts[b] parts with the same tile
  // boundaries; CTA c of episode b's block of H * kparts[b] CTAs reads part c / H of head c % H
  uint16_t kparts[WAM_MAX_EPISODE_FRAMES];
  float* ws_part;     // partial (O, m, l) slots [B*H][max_parts][32*128 + 64]
  int* ws_count;      // arrival tickets [B*H]; zero between calls
  int32_t ksplit;     // CTAs (one thread-block cluster) per (episode, head) of the cluster read
  int32_t fused_ready;  // the fused pair is not written by the previous kernel on the stream
  float scale_log2;
  int* err;
  // NVFP4 fused pair (wam_action_attn_nvfp4; null otherwise): head-major codes [B, H, N, 64],
  // E4M3 block scales [B, H, N, 8] and the device tensor scale of K and of V
  const uint8_t* k_codes;
  const uint8_t* k_scales;
  const uint8_t* v_codes;
  const uint8_t* v_scales;
  const float* k_sg;
  const float* v_sg;
  FrameLists fl;
};

// NVFP4 encoding of n fused tensors (nvfp4.cu).  ws holds kNvfp4MaxSlices |x| maxima per
// tensor between the two launches.
constexpr int kNvfp4MaxSlices = 1024;
struct Nvfp4Args {
  const void* src[WAM_MAX_NVFP4_TENSORS];  // bf16 [B, N, H, D]
  void* codes[WAM_MAX_NVFP4_TENSORS];      // [B, H, N, D / 2]
  void* scales[WAM_MAX_NVFP4_TENSORS];     // [B, H, N, D / 16]
  float* s_g;                              // [n]
  float* ws;                               // [n][kNvfp4MaxSlices]
  int32_t n, B, H, D, T, F, slices;
  int64_t frame_elems;                     // T * H * D
  FrameLists fl;                           // items: the valid (b, f) frames
};

struct CopyArgs {
  const void* src[WAM_MAX_COPY_TENSORS];
  void* dst[WAM_MAX_COPY_TENSORS];
  int32_t n, B;
  int64_t ep_vec;    // 16-byte vectors of one episode's tensor (F*T*H*D*es / 16)
  int64_t src_vec;   // first vector copied within an episode
  int64_t dst_vec;
  int64_t n_vec;     // vectors copied per (tensor, episode)
};

struct FuseArgs {
  const void* k[WAM_MAX_FUSE_LAYERS];
  const void* v[WAM_MAX_FUSE_LAYERS];
  float w[WAM_MAX_FUSE_LAYERS];
  int32_t n_layers;
  void* fk;
  void* fv;
  int64_t frame_elems;  // T*H*D
  int32_t F;
  FrameLists fl;        // items: (b, f) frames to fuse
};

// ---------------------------------------------------------------------------------------
// Element access
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

constexpr uint32_t kWaitSpinLimit = 1u << 24;  // try_wait rounds before a wait gives up
// A warp that polls several barriers with test_wait and found none of them ready pauses for a
// moment (at most twice this many nanoseconds), so that the warps sharing its scheduler keep
// their issue slots.
constexpr unsigned kPollPauseNs = 32;
__device__ __forceinline__ void poll_pause() { __nanosleep(kPollPauseNs); }

// ---------------------------------------------------------------------------------------
// PTX wrappers: shared-memory addresses, mbarriers, TMA, ldmatrix, mma.sync
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// The first 1024-byte-aligned byte of dynamic shared memory, found by pointer arithmetic on the
// shared array itself: the compiler then keeps every access through the result in the shared
// state space, where a round trip through an integer would leave a generic pointer.
__device__ __forceinline__ uint8_t* smem_align1024(uint8_t* raw) {
  return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Programmatic dependent launch: a kernel launched with programmatic stream serialization
// may start while the previous kernel on its stream is still running.  It waits here (until
// that grid has completed and its memory is visible) before its first global memory access,
// and lets the next kernel start launching as early as possible.  Both are no-ops for a kernel
// launched without the attribute.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Non-blocking test of a phase (mbarrier.try_wait may suspend the thread for a while when the
// phase is not complete; a thread that polls several barriers uses this instead).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false if the phase never flips within `limit` polls; the caller then
// records WAM_ERR_TIMEOUT in the device error word (args.err) and leaves without waiting
// further.  The kernels use kWaitSpinLimit; wam_debug_wait_timeout passes a short limit.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_wait_bounded(bar, parity, kWaitSpinLimit);
}

// 4-D tiled TMA load global -> shared, completion counted on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A * B + D, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A * B + D, m16n8k8, tf32 inputs (b32 registers), fp32 accumulators.
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp32 -> tf32, round to nearest (ties away from zero).
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// The two bf16 halves of a packed register widened to fp32 bit patterns (exact as tf32).
__device__ __forceinline__ uint32_t bf16_lo_bits(uint32_t r) { return r << 16; }
__device__ __forceinline__ uint32_t bf16_hi_bits(uint32_t r) { return r & 0xffff0000u; }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of element (row, col) in a [rows x 128] bf16 tile stored as two 128B-swizzled
// halves of [rows x 64] (the layout a TMA box of 64 x rows with SWIZZLE_128B writes).
template <int ROWS>
__device__ __forceinline__ uint32_t swz128(int row, int col) {
  const int half = col >> 6, cc = col & 63;
  return uint32_t(half * ROWS * 128 + row * 128 + ((((cc >> 3) ^ (row & 7))) << 4) + ((cc & 7) << 1));
}

}  // namespace wam
