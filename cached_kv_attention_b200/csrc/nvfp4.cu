// NVFP4 encoding of a fused K or V cache ("Long-WAM: 机器人操作模型的长历史..." §四: the
// LongLive-2.0 stack quantises its KV cache block-wise to NVFP4, about 3.6x smaller; the
// format is NVIDIA's public NVFP4): E2M1 elements, one E4M3 scale per 16 consecutive elements
// along D, one fp32 scale per tensor s_g = amax / (6 * 448).
//
// Two launches over n tensors at once: the first takes |x| maxima of slices of each tensor's
// non-padding frames into the workspace; the second reduces them to the tensor's amax, and
// encodes one 16-element block per thread.  Every code decision is taken in fp32 in the order
//   s_g = amax / 2688;  s_b = e4m3(amax_b / (6 s_g));  y = x / (e4m3 value of s_b * s_g);
//   code = e2m1(y)
// with IEEE division and products and the conversions' round-to-nearest-even, saturating to
// the largest finite value; a negative value that rounds to zero gets the +0 code.
// Output layout, head-major so that one 128-key tile of one head is one contiguous run:
//   codes  [B, H, N, D / 2] bytes, element 2i in the low nibble of byte i
//   scales [B, H, N, D / 16] E4M3 codes
#include "launch.h"

namespace wam {
namespace {

constexpr int kThreadsQ = 256;

// |x| maxima over slices of every tensor's valid frames; one slice per CTA (blockIdx.x) of
// tensor blockIdx.y.  A slice is a contiguous range of 16-byte vectors of the valid frames.
__global__ void __launch_bounds__(kThreadsQ) nvfp4_amax_kernel(const __grid_constant__ Nvfp4Args a) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int y = blockIdx.y;
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.src[y]);
  const int64_t frame_vec = a.frame_elems / 8;  // 16-byte vectors per frame
  const int64_t total = int64_t(a.fl.n_items) * frame_vec;
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  const int64_t v0 = per * blockIdx.x, v1 = v0 + per < total ? v0 + per : total;
  float mx = 0.f;
  for (int64_t v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
    const int64_t item = v / frame_vec, in = v % frame_vec;
    const uint32_t it = a.fl.item[item];
    const int64_t off = (int64_t(item_b(it)) * a.F + item_f(it)) * a.frame_elems + in * 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(x + off);
    const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
    for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(__bfloat162float(e[i])));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  __shared__ float wmax[kThreadsQ / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int i = 0; i < kThreadsQ / 32; ++i) m = fmaxf(m, wmax[i]);
    a.ws[int64_t(y) * kNvfp4MaxSlices + blockIdx.x] = m;
  }
}

// E2M1 codes of two fp32 values (first in the low nibble), +0 for a value that rounds to zero.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %2, %1; cvt.u32.u8 %0, t; }"
      : "=r"(r)
      : "f"(lo), "f"(hi));
  if ((r & 0x07u) == 0) r &= 0xF0u;
  if ((r & 0x70u) == 0) r &= 0x0Fu;
  return r;
}
// E4M3 code of a non-negative fp32 value, and the value of an E4M3 code.
__device__ __forceinline__ uint32_t e4m3_code(float v) {
  uint32_t r;
  asm("{ .reg .b16 t; cvt.rn.satfinite.e4m3x2.f32 t, %1, %1; cvt.u32.u16 %0, t; }" : "=r"(r) : "f"(v));
  return r & 0xFFu;
}
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h2;
  // both bytes hold the code, so both halves of the result hold its value
  asm("{ .reg .b16 c; cvt.u16.u32 c, %1; cvt.rn.f16x2.e4m3x2 %0, c; }" : "=r"(h2) : "r"(code | (code << 8)));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// One 16-element block per thread: (valid frame item, token, head, block j of D / 16).
__global__ void __launch_bounds__(kThreadsQ) nvfp4_encode_kernel(const __grid_constant__ Nvfp4Args a) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int y = blockIdx.y;
  __shared__ float s_amax;
  if (threadIdx.x < 32) {
    float m = 0.f;
    for (int i = threadIdx.x; i < a.slices; i += 32) m = fmaxf(m, a.ws[int64_t(y) * kNvfp4MaxSlices + i]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) s_amax = m;
  }
  __syncthreads();
  const float s_g = __fdiv_rn(s_amax, 2688.f);  // 6 * 448
  if (blockIdx.x == 0 && threadIdx.x == 0) a.s_g[y] = s_g;
  const float six_sg = __fmul_rn(6.f, s_g);
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.src[y]);
  uint8_t* codes = static_cast<uint8_t*>(a.codes[y]);
  uint8_t* scales = static_cast<uint8_t*>(a.scales[y]);
  const int nblk = a.D / 16;
  const int64_t per_frame = int64_t(a.T) * a.H * nblk;  // blocks per frame
  const int64_t total = int64_t(a.fl.n_items) * per_frame;
  const int64_t N = int64_t(a.F) * a.T;
  for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < total;
       g += int64_t(gridDim.x) * blockDim.x) {
    const int64_t item = g / per_frame;
    int64_t r = g % per_frame;
    const int j = int(r % nblk);
    r /= nblk;
    const int h = int(r % a.H);
    const int t = int(r / a.H);
    const uint32_t it = a.fl.item[item];
    const int b = item_b(it);
    const int64_t tok = int64_t(item_f(it)) * a.T + t;
    const __nv_bfloat16* src = x + ((int64_t(b) * N + tok) * a.H + h) * a.D + 16 * j;
    const uint4 r0 = *reinterpret_cast<const uint4*>(src), r1 = *reinterpret_cast<const uint4*>(src + 8);
    float v[16];
    {
      const __nv_bfloat16* e0 = reinterpret_cast<const __nv_bfloat16*>(&r0);
      const __nv_bfloat16* e1 = reinterpret_cast<const __nv_bfloat16*>(&r1);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __bfloat162float(e0[i]), v[8 + i] = __bfloat162float(e1[i]);
    }
    uint32_t sb = 0, packed[2] = {0u, 0u};
    if (s_g > 0.f) {
      float amax_b = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(v[i]));
      sb = e4m3_code(__fdiv_rn(amax_b, six_sg));
      const float scale = __fmul_rn(e4m3_value(sb), s_g);
      if (scale > 0.f) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t c = e2m1x2(__fdiv_rn(v[2 * i], scale), __fdiv_rn(v[2 * i + 1], scale));
          packed[i >> 2] |= c << (8 * (i & 3));
        }
      }
    }
    const int64_t row = (int64_t(b) * a.H + h) * N + tok;  // head-major row of (b, h, token)
    *reinterpret_cast<uint2*>(codes + row * (a.D / 2) + 8 * j) = make_uint2(packed[0], packed[1]);
    scales[row * nblk + j] = static_cast<uint8_t>(sb);
  }
}

}  // namespace

cudaError_t launch_nvfp4_encode(Nvfp4Args& a, cudaStream_t s) {
  if (a.fl.n_items == 0 || a.n == 0) return cudaSuccess;
  const int64_t vec = int64_t(a.fl.n_items) * (a.frame_elems / 8);
  int slices = int((vec + kThreadsQ * 8 - 1) / (kThreadsQ * 8));  // >= 8 vectors per thread
  if (slices > kNvfp4MaxSlices) slices = kNvfp4MaxSlices;
  if (slices < 1) slices = 1;
  a.slices = slices;
  cudaError_t e = launch_pdl(nvfp4_amax_kernel, dim3(unsigned(slices), unsigned(a.n)), dim3(kThreadsQ), 0, s, 0, a);
  if (e != cudaSuccess) return e;
  const int64_t blocks = int64_t(a.fl.n_items) * a.T * a.H * (a.D / 16);
  int64_t g = (blocks + kThreadsQ - 1) / kThreadsQ;
  if (g > 1184) g = 1184;  // 8 per SM on 148 SMs; the kernel strides over the rest
  return launch_pdl(nvfp4_encode_kernel, dim3(unsigned(g), unsigned(a.n)), dim3(kThreadsQ), 0, s, 0, a);
}

}  // namespace wam
