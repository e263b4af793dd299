// CUDA-core kernels: Euler step, cache store + fusion epilogue, standalone Interval
// KV-Fusion, the video mask export, and the fp32-accumulating attention path that serves
// every shape without a tensor-core kernel (the fp32 workload among them).
#include "launch.h"

namespace wam {

// ------------------------------------------------------------------------------ vectors
template <typename E, int W> struct Vec;
template <> struct Vec<float, 4> { using T = float4; };
template <> struct Vec<float, 2> { using T = float2; };
template <> struct Vec<__nv_bfloat16, 8> { using T = uint4; };
template <> struct Vec<__nv_bfloat16, 4> { using T = uint2; };
template <> struct Vec<__nv_bfloat16, 2> { using T = uint32_t; };

template <typename E, int W>
__device__ __forceinline__ void vload(const E* p, float (&o)[W]) {
  typename Vec<E, W>::T raw = *reinterpret_cast<const typename Vec<E, W>::T*>(p);
  const E* e = reinterpret_cast<const E*>(&raw);
#pragma unroll
  for (int i = 0; i < W; ++i) o[i] = to_f(e[i]);
}
template <typename E, int W>
__device__ __forceinline__ void vstore(E* p, const float (&x)[W]) {
  typename Vec<E, W>::T raw;
  E* e = reinterpret_cast<E*>(&raw);
#pragma unroll
  for (int i = 0; i < W; ++i) e[i] = from_f<E>(x[i]);
  *reinterpret_cast<typename Vec<E, W>::T*>(p) = raw;
}

static int grid_for(int64_t work, int per_block, int cap) {
  int64_t g = (work + per_block - 1) / per_block;
  if (g > cap) g = cap;
  return g < 1 ? 1 : int(g);
}

// ------------------------------------------------------------------------------ bounded wait
// A wait that runs out, on purpose: one warp waits on an mbarrier that nothing arrives on,
// with a short poll limit, and reports WAM_ERR_TIMEOUT through the device error word as the
// attention kernels do when one of their waits gives up.  It holds no TMA, tensor-core or
// tensor-memory work, so giving up leaves nothing in flight.
__global__ void wait_timeout_kernel(uint32_t polls, int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const bool done = mbar_wait_bounded(&bar, 0, polls);  // phase 0 never completes
  if (!__any_sync(0xffffffffu, done) && threadIdx.x == 0 && err)
    atomicExch(err, int(WAM_ERR_TIMEOUT));
}

cudaError_t launch_wait_timeout(uint32_t polls, int* err, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(polls, err);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------ Euler
__global__ void euler_kernel(int64_t n, float* __restrict__ x, const float* __restrict__ v,
                             float dsigma) {
  grid_dependency_wait();  // programmatic dependent launch: inputs ready from here on
  grid_launch_dependents();
  const int64_t n4 = n >> 2;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const int64_t i0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t i = i0; i < n4; i += stride) {
    float4 a = reinterpret_cast<float4*>(x)[i];
    const float4 b = reinterpret_cast<const float4*>(v)[i];
    a.x = fmaf(dsigma, b.x, a.x);
    a.y = fmaf(dsigma, b.y, a.y);
    a.z = fmaf(dsigma, b.z, a.z);
    a.w = fmaf(dsigma, b.w, a.w);
    reinterpret_cast<float4*>(x)[i] = a;
  }
  for (int64_t i = (n4 << 2) + i0; i < n; i += stride) x[i] = fmaf(dsigma, v[i], x[i]);
}

cudaError_t launch_euler(int64_t n, float* x, const float* v, float dsigma, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  return launch_pdl(euler_kernel, dim3(grid_for((n + 3) / 4, 256, 148 * 16)), dim3(256), 0, s, 0, n, x, v, dsigma);
}

// ------------------------------------------------------------------------------ frame copies
// blockIdx.y = tensor pair j * B + episode b; a grid-stride loop over the 16-byte vectors of
// the copied frames (contiguous within an episode).
__global__ void copy_frames_kernel(const __grid_constant__ CopyArgs a) {
  grid_dependency_wait();  // programmatic dependent launch: inputs ready from here on
  grid_launch_dependents();
  const int j = int(blockIdx.y) / a.B, b = int(blockIdx.y) % a.B;
  const uint4* src = static_cast<const uint4*>(a.src[j]) + int64_t(b) * a.ep_vec + a.src_vec;
  uint4* dst = static_cast<uint4*>(a.dst[j]) + int64_t(b) * a.ep_vec + a.dst_vec;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.n_vec;
       i += int64_t(gridDim.x) * blockDim.x)
    dst[i] = __ldcs(src + i);  // streamed once: evict-first
}

cudaError_t launch_copy_frames(const CopyArgs& a, cudaStream_t s) {
  if (a.n_vec == 0) return cudaSuccess;
  const int64_t pairs = int64_t(a.n) * a.B;
  const int64_t per_pair = (a.n_vec + 255) / 256;
  const int64_t want = (148 * 8 + pairs - 1) / pairs;  // ~8 blocks per SM over all pairs
  const unsigned gx = unsigned(per_pair < want ? per_pair : (want < 1 ? 1 : want));
  return launch_pdl(copy_frames_kernel, dim3(gx, unsigned(pairs)), dim3(256), 0, s, 0, a);
}

// ------------------------------------------------------------------------------ store + fuse
// Copies the new K/V of every valid query frame into the cache and applies the fusion
// epilogue (acc = w K | acc += w K | fused = round(acc + w K)).  grid (chunks, items, 2).
template <typename E, int W>
__global__ void store_fuse_kernel(const __grid_constant__ PrefillArgs a, int64_t frame_elems) {
  const uint32_t it = a.fl.item[blockIdx.y];
  const int b = item_b(it), f = item_f(it), kv = blockIdx.z;
  const int64_t qtok = int64_t(a.f_end - a.f_begin) * a.T, N = int64_t(a.F) * a.T;
  const int64_t row = frame_elems / a.T;  // H * D
  const E* src = static_cast<const E*>(kv ? a.v_new : a.k_new) +
                 (int64_t(b) * qtok + int64_t(f - a.f_begin) * a.T) * row;
  const int64_t dst = (int64_t(b) * N + int64_t(f) * a.T) * row;
  E* store = a.k_store ? static_cast<E*>(kv ? a.v_store : a.k_store) + dst : nullptr;
  float* acc = (a.fuse_on && (kv ? a.acc_v : a.acc_k)) ? (kv ? a.acc_v : a.acc_k) + dst : nullptr;
  E* fused = (a.fuse_on && a.fuse_last) ? static_cast<E*>(kv ? a.fused_v : a.fused_k) + dst
                                        : nullptr;
  const int64_t nv = frame_elems / W;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nv;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t e = i * W;
    float x[W];
    vload<E, W>(src + e, x);
    if (store) vstore<E, W>(store + e, x);
    if (a.fuse_on) {
      float s[W];
      if (a.fuse_first) {
#pragma unroll
        for (int j = 0; j < W; ++j) s[j] = a.fuse_w * x[j];
      } else {
#pragma unroll
        for (int j = 0; j < W; j += 4) {
          const float4 p = *reinterpret_cast<const float4*>(acc + e + j);
          s[j] = fmaf(a.fuse_w, x[j], p.x);
          s[j + 1] = fmaf(a.fuse_w, x[j + 1], p.y);
          s[j + 2] = fmaf(a.fuse_w, x[j + 2], p.z);
          s[j + 3] = fmaf(a.fuse_w, x[j + 3], p.w);
        }
      }
      if (a.fuse_last) {
        vstore<E, W>(fused + e, s);
      } else {
#pragma unroll
        for (int j = 0; j < W; j += 4)
          *reinterpret_cast<float4*>(acc + e + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
      }
    }
  }
}

cudaError_t launch_store_fuse(const PrefillArgs& a, int D, bool bf16, cudaStream_t s) {
  if (a.fl.n_items == 0 || (!a.k_store && !a.fuse_on)) return cudaSuccess;
  const int64_t fe = int64_t(a.T) * a.H * D;
  const int W = bf16 ? 8 : 4;
  dim3 grid(grid_for(fe / W, 256, 64), a.fl.n_items, 2);
  if (bf16)
    store_fuse_kernel<__nv_bfloat16, 8><<<grid, 256, 0, s>>>(a, fe);
  else
    store_fuse_kernel<float, 4><<<grid, 256, 0, s>>>(a, fe);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------ fusion
// fused = round(sum_j w_j layer_j) in fp32 over the listed (episode, frame) runs.
template <typename E, int W>
__global__ void fuse_kernel(const __grid_constant__ FuseArgs a) {
  const uint32_t it = a.fl.item[blockIdx.y];
  const int b = item_b(it), f = item_f(it), kv = blockIdx.z;
  const int64_t base = (int64_t(b) * a.F + f) * a.frame_elems;
  E* out = static_cast<E*>(kv ? a.fv : a.fk) + base;
  const int64_t nv = a.frame_elems / W;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nv;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t e = i * W;
    float s[W];
#pragma unroll
    for (int j = 0; j < W; ++j) s[j] = 0.f;
    for (int l = 0; l < a.n_layers; ++l) {
      float x[W];
      vload<E, W>(static_cast<const E*>(kv ? a.v[l] : a.k[l]) + base + e, x);
#pragma unroll
      for (int j = 0; j < W; ++j) s[j] = fmaf(a.w[l], x[j], s[j]);
    }
    vstore<E, W>(out + e, s);
  }
}

cudaError_t launch_fuse(const FuseArgs& a, int D, bool bf16, cudaStream_t s) {
  if (a.fl.n_items == 0) return cudaSuccess;
  const int W = bf16 ? 8 : 4;
  dim3 grid(grid_for(a.frame_elems / W, 256, 64), a.fl.n_items, 2);
  if (bf16)
    fuse_kernel<__nv_bfloat16, 8><<<grid, 256, 0, s>>>(a);
  else
    fuse_kernel<float, 4><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
  (void)D;
}

// ------------------------------------------------------------------------------ mask export
// The video predicate exactly as the attention kernels apply it: a query frame reads the
// first nk entries of its episode's valid-frame list, and only query frames with a work item
// produce output.
__global__ void debug_mask_kernel(const __grid_constant__ PrefillArgs a, uint8_t* mask) {
  const int64_t Q = int64_t(a.f_end - a.f_begin) * a.T, K = int64_t(a.f_end) * a.T;
  const int64_t total = int64_t(a.B) * Q * K;
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int b = int(idx / (Q * K));
    const int fq = a.f_begin + int((idx / K) % Q) / a.T;
    const int fk = int(idx % K) / a.T;
    uint8_t ok = 0;
    for (int j = 0; j < a.fl.n_items; ++j) {
      const uint32_t it = a.fl.item[j];
      if (item_b(it) != b || item_f(it) != fq) continue;
      for (int u = 0; u < item_nk(it); ++u)
        if (a.fl.vlist[b * a.F + u] == fk) ok = 1;
    }
    mask[idx] = ok;
  }
}

cudaError_t launch_debug_mask(const PrefillArgs& a, uint8_t* mask, cudaStream_t s) {
  const int64_t total = int64_t(a.B) * (a.f_end - a.f_begin) * a.T * int64_t(a.f_end) * a.T;
  if (total == 0) return cudaSuccess;
  debug_mask_kernel<<<grid_for(total, 256, 148 * 8), 256, 0, s>>>(a, mask);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------ attention
// One warp per query row; each lane holds D/32 contiguous elements; the dot product is a
// warp-shuffle reduction and the softmax is online in fp32 (exp2 of log2e-scaled logits).
template <int PER>
__device__ __forceinline__ float warp_dot(const float (&q)[PER], const float (&k)[PER]) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) s = fmaf(q[i], k[i], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

template <int PER>
struct RowState {
  float m = -INFINITY, l = 0.f, acc[PER];
  __device__ RowState() {
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  }
  __device__ __forceinline__ void add(float s, const float (&v)[PER]) {
    const float mn = fmaxf(m, s);
    const float alpha = exp2f(m - mn), p = exp2f(s - mn);
    l = fmaf(l, alpha, p);
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = fmaf(acc[i], alpha, p * v[i]);
    m = mn;
  }
};

template <typename E, int D>
__device__ __forceinline__ void store_row(void* o, bool o_f32, int64_t off, const float (&acc)[D / 32],
                                          float inv_l) {
  constexpr int PER = D / 32;
  float x[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) x[i] = acc[i] * inv_l;
  if (o_f32)
    vstore<float, PER>(static_cast<float*>(o) + off, x);
  else
    vstore<E, PER>(static_cast<E*>(o) + off, x);
}

constexpr int kSimtRows = 16;  // query rows per CTA (4 warps x 4 rows)

template <typename E, int D>
__global__ void __launch_bounds__(128) prefill_simt_kernel(const __grid_constant__ PrefillArgs a) {
  constexpr int PER = D / 32;
  const int nqc = (a.T + kSimtRows - 1) / kSimtRows;
  const uint32_t it = a.fl.item[blockIdx.x / nqc];
  const int qc = blockIdx.x % nqc, h = blockIdx.y;
  const int b = item_b(it), f = item_f(it), nk = item_nk(it);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t qtok = int64_t(a.f_end - a.f_begin) * a.T, N = int64_t(a.F) * a.T;
  const E* Q = static_cast<const E*>(a.q);
  for (int r = warp; r < kSimtRows; r += 4) {
    const int i = qc * kSimtRows + r;
    if (i >= a.T) break;
    const int64_t tq = int64_t(b) * qtok + int64_t(f - a.f_begin) * a.T + i;
    float q[PER];
    vload<E, PER>(Q + (tq * a.H + h) * D + lane * PER, q);
    RowState<PER> st;
    for (int u = 0; u < nk; ++u) {
      const int fk = a.fl.vlist[b * a.F + u];
      const bool old = fk < a.f_begin;
      const E* K = static_cast<const E*>(old ? a.k_cache : a.k_new);
      const E* V = static_cast<const E*>(old ? a.v_cache : a.v_new);
      const int64_t t0 = old ? int64_t(b) * N + int64_t(fk) * a.T
                             : int64_t(b) * qtok + int64_t(fk - a.f_begin) * a.T;
      for (int j = 0; j < a.T; ++j) {
        const int64_t off = ((t0 + j) * a.H + h) * D + lane * PER;
        float k[PER], v[PER];
        vload<E, PER>(K + off, k);
        vload<E, PER>(V + off, v);
        st.add(warp_dot<PER>(q, k) * a.scale_log2, v);
      }
    }
    store_row<E, D>(a.o, a.o_f32, (tq * a.H + h) * D + lane * PER, st.acc, 1.f / st.l);
  }
}

cudaError_t launch_prefill_simt(const PrefillArgs& a, int D, bool bf16, cudaStream_t s) {
  if (a.fl.n_items == 0) return cudaSuccess;
  const int nqc = (a.T + kSimtRows - 1) / kSimtRows;
  dim3 grid(a.fl.n_items * nqc, a.H);
  if (bf16) {
    if (D == 128) prefill_simt_kernel<__nv_bfloat16, 128><<<grid, 128, 0, s>>>(a);
    else prefill_simt_kernel<__nv_bfloat16, 64><<<grid, 128, 0, s>>>(a);
  } else {
    if (D == 128) prefill_simt_kernel<float, 128><<<grid, 128, 0, s>>>(a);
    else prefill_simt_kernel<float, 64><<<grid, 128, 0, s>>>(a);
  }
  return cudaGetLastError();
}

template <typename E, int D>
__global__ void __launch_bounds__(128) action_simt_kernel(const __grid_constant__ ActionArgs a) {
  constexpr int PER = D / 32;
  const int b = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t N = int64_t(a.F) * a.T;
  const E* Qa = static_cast<const E*>(a.qa);
  const E* Ka = static_cast<const E*>(a.ka);
  const E* Va = static_cast<const E*>(a.va);
  for (int i = warp; i < a.n_act; i += 4) {
    const int64_t tq = int64_t(b) * a.n_act + i;
    float q[PER];
    vload<E, PER>(Qa + (tq * a.H + h) * D + lane * PER, q);
    RowState<PER> st;
    if (a.with_video) {
      const E* K = static_cast<const E*>(a.fk);
      const E* V = static_cast<const E*>(a.fv);
      for (int u = 0; u < a.fl.nvalid[b]; ++u) {
        const int64_t t0 = int64_t(b) * N + int64_t(a.fl.vlist[b * a.F + u]) * a.T;
        for (int j = 0; j < a.T; ++j) {
          const int64_t off = ((t0 + j) * a.H + h) * D + lane * PER;
          float k[PER], v[PER];
          vload<E, PER>(K + off, k);
          vload<E, PER>(V + off, v);
          st.add(warp_dot<PER>(q, k) * a.scale_log2, v);
        }
      }
    }
    for (int j = 0; j < a.n_act; ++j) {
      const int64_t off = ((int64_t(b) * a.n_act + j) * a.H + h) * D + lane * PER;
      float k[PER], v[PER];
      vload<E, PER>(Ka + off, k);
      vload<E, PER>(Va + off, v);
      st.add(warp_dot<PER>(q, k) * a.scale_log2, v);
    }
    store_row<E, D>(a.o, a.o_f32, (tq * a.H + h) * D + lane * PER, st.acc, 1.f / st.l);
  }
}

cudaError_t launch_action_simt(const ActionArgs& a, int D, bool bf16, cudaStream_t s) {
  dim3 grid(a.B, a.H);
  if (bf16) {
    if (D == 128) action_simt_kernel<__nv_bfloat16, 128><<<grid, 128, 0, s>>>(a);
    else action_simt_kernel<__nv_bfloat16, 64><<<grid, 128, 0, s>>>(a);
  } else {
    if (D == 128) action_simt_kernel<float, 128><<<grid, 128, 0, s>>>(a);
    else action_simt_kernel<float, 64><<<grid, 128, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace wam
