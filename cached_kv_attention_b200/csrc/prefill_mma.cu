// Block-causal video prefill on mma.sync tensor-core tiles (bf16, D = 128, T % 128 == 0).
//
// One CTA computes 128 query tokens of one (episode, frame, head) against every key tile the
// block-causal predicate allows ("Long-WAM: Scaling the Context of World-Action Models |
// Summary" §3.1-3.2: a video query reads its own and earlier visual blocks).  Because T is a
// multiple of 128, every tile is wholly visible or wholly masked: the host work list already
// holds only visible key frames (padding frames dropped, later blocks cut off), so the kernel
// applies no element mask.  Keys of frames below f_begin come from the layer's cache, the
// others from the call's new K/V.
//
// While the CTA's own 128 tokens of K/V are resident in shared memory it stores them into
// the cache and folds them into the Interval KV-Fusion accumulator ("世界模型之Faster-WAM详解"
// §3.3), so the per-layer K/V is never re-read from HBM for fusion.
//
// Warp roles: warps 0-7 consume (16 query rows each), warp 8 lane 0 issues TMA loads into a
// 3-stage K/V ring (full/empty mbarriers, bounded waits).
#include "launch.h"

namespace wam {
namespace {

constexpr int kBM = 128, kBN = 64;
constexpr int kStages = 3;
constexpr int kConsumers = 8;
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kQBytes = kBM * 128 * 2;
constexpr int kTileBytes = kBN * 128 * 2;
constexpr int kSmemBytes = 1024 + kQBytes + kStages * 2 * kTileBytes + 256;

struct PrefillMaps {
  CUtensorMap q, kn, vn, kc, vc;
};

// Store (and fold into the fusion accumulator) one resident 64-token K or V tile.
__device__ __forceinline__ void store_fuse_tile(const PrefillArgs& a, const uint8_t* tile,
                                                const void* store_base, float* acc_base,
                                                void* fused_base, int64_t row0, int h, int tid) {
  for (int c = tid; c < kBN * 16; c += kConsumers * 32) {
    const int r = c >> 4, cc = (c & 15) * 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(tile + swz128<kBN>(r, cc));
    const int64_t off = ((row0 + r) * a.H + h) * 128 + cc;
    if (store_base)
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(store_base)) + off) = raw;
    if (a.fuse_on) {
      const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&raw);
      float s[8];
      if (a.fuse_first) {
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] = a.fuse_w * __bfloat162float(x[j]);
      } else {
        const float4 p0 = *reinterpret_cast<const float4*>(acc_base + off);
        const float4 p1 = *reinterpret_cast<const float4*>(acc_base + off + 4);
        const float p[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] = fmaf(a.fuse_w, __bfloat162float(x[j]), p[j]);
      }
      if (a.fuse_last) {
        uint4 u;
        u.x = pack_bf16(s[0], s[1]), u.y = pack_bf16(s[2], s[3]);
        u.z = pack_bf16(s[4], s[5]), u.w = pack_bf16(s[6], s[7]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(fused_base) + off) = u;
      } else {
        *reinterpret_cast<float4*>(acc_base + off) = make_float4(s[0], s[1], s[2], s[3]);
        *reinterpret_cast<float4*>(acc_base + off + 4) = make_float4(s[4], s[5], s[6], s[7]);
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_mma_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ PrefillMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = base;
  uint8_t* sk[kStages];
  uint8_t* sv[kStages];
  for (int i = 0; i < kStages; ++i) {
    sk[i] = base + kQBytes + i * 2 * kTileBytes;
    sv[i] = sk[i] + kTileBytes;
  }
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kQBytes + kStages * 2 * kTileBytes);
  uint64_t* empty = full + kStages;
  uint64_t* qbar = empty + kStages;

  const int QT = a.T / kBM;
  const int h = int(blockIdx.x % a.H);
  const int rest = int(blockIdx.x / a.H);
  const int qt = rest % QT;
  const uint32_t it = a.fl.item[rest / QT];
  const int b = item_b(it), f = item_f(it), nk = item_nk(it);
  const int tpf = a.T / kBN;
  const int n_tiles = nk * tpf;
  const int qtok0 = (f - a.f_begin) * a.T + qt * kBM;  // first query row of the call
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool do_store = a.k_store != nullptr || a.fuse_on;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumers);
    }
    mbar_init(qbar, 1);
    fence_barrier_init();
  }
  __syncthreads();

  bool bad = false;
  if (warp == kConsumers) {
    if (lane == 0) {
      mbar_arrive_expect_tx(qbar, kQBytes);
      tma_load_4d(sq, &maps.q, qbar, 0, h, qtok0, b);
      tma_load_4d(sq + kQBytes / 2, &maps.q, qbar, 64, h, qtok0, b);
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int st = i % kStages;
        if (i >= kStages && !mbar_wait(&empty[st], ((i / kStages) - 1) & 1)) { bad = true; break; }
        const int fk = a.fl.vlist[b * a.F + i / tpf];
        const int j = i % tpf;
        const bool old = fk < a.f_begin;
        const CUtensorMap* mk = old ? &maps.kc : &maps.kn;
        const CUtensorMap* mv = old ? &maps.vc : &maps.vn;
        const int tok = (old ? fk : fk - a.f_begin) * a.T + j * kBN;
        mbar_arrive_expect_tx(&full[st], 2 * kTileBytes);
        tma_load_4d(sk[st], mk, &full[st], 0, h, tok, b);
        tma_load_4d(sk[st] + kTileBytes / 2, mk, &full[st], 64, h, tok, b);
        tma_load_4d(sv[st], mv, &full[st], 0, h, tok, b);
        tma_load_4d(sv[st] + kTileBytes / 2, mv, &full[st], 64, h, tok, b);
        issued = i + 1;
      }
      for (int i = max(0, issued - kStages); i < issued; ++i)
        if (!mbar_wait(&full[i % kStages], (i / kStages) & 1)) break;
      if (!mbar_wait(qbar, 0)) bad = true;
    }
  } else {
    const int g = lane >> 2, t = lane & 3;
    float oacc[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    uint32_t qf[8][4];
    if (!mbar_wait(qbar, 0)) bad = true;
    if (!bad) {
      const uint32_t qb = smem_u32(sq);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        ldsm_x4(qb + swz128<kBM>(16 * warp + (lane & 15), 16 * kk + (lane >> 4) * 8), qf[kk][0],
                qf[kk][1], qf[kk][2], qf[kk][3]);
    }
    const float c = a.scale_log2;
    const int64_t N = int64_t(a.F) * a.T;
    for (int i = 0; i < n_tiles && !bad; ++i) {
      const int st = i % kStages;
      if (!mbar_wait(&full[st], (i / kStages) & 1)) { bad = true; break; }
      const uint32_t kb = smem_u32(sk[st]), vb = smem_u32(sv[st]);
      float s[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + swz128<kBN>(16 * p + (lane & 7) + (lane >> 4) * 8, 16 * kk + ((lane >> 3) & 1) * 8),
                  b0, b1, b2, b3);
          mma_bf16(s[2 * p], qf[kk], b0, b1);
          mma_bf16(s[2 * p + 1], qf[kk], b2, b3);
        }
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
        mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0 * c), mn1 = fmaxf(m1, mx1 * c);
      const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        s[j][0] = exp2f(fmaf(s[j][0], c, -mn0));
        s[j][1] = exp2f(fmaf(s[j][1], c, -mn0));
        s[j][2] = exp2f(fmaf(s[j][2], c, -mn1));
        s[j][3] = exp2f(fmaf(s[j][3], c, -mn1));
        rs0 += s[j][0] + s[j][1];
        rs1 += s[j][2] + s[j][3];
      }
      l0 = fmaf(l0, al0, rs0);
      l1 = fmaf(l1, al1, rs1);
      m0 = mn0, m1 = mn1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        oacc[j][0] *= al0, oacc[j][1] *= al0, oacc[j][2] *= al1, oacc[j][3] *= al1;
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vb + swz128<kBN>(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8, 16 * p + (lane >> 4) * 8),
                    b0, b1, b2, b3);
          mma_bf16(oacc[2 * p], pa, b0, b1);
          mma_bf16(oacc[2 * p + 1], pa, b2, b3);
        }
      }
      // Own tokens resident: store them into the cache and fold them into the fusion.
      if (do_store) {
        const int fk = a.fl.vlist[b * a.F + i / tpf];
        const int j = i % tpf;
        if (fk == f && (j >> 1) == qt) {
          const int64_t row0 = int64_t(b) * N + int64_t(f) * a.T + j * kBN;
          const int tid = threadIdx.x;
          store_fuse_tile(a, sk[st], a.k_store, a.acc_k, a.fused_k, row0, h, tid);
          store_fuse_tile(a, sv[st], a.v_store, a.acc_v, a.fused_v, row0, h, tid);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = 1.f / l0, i1 = 1.f / l1;
    const int64_t qtok = int64_t(a.f_end - a.f_begin) * a.T;
    const int64_t r0 = int64_t(b) * qtok + qtok0 + 16 * warp + g, r1 = r0 + 8;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int col = 8 * j + 2 * t;
      if (a.o_f32) {
        float* o = static_cast<float*>(a.o);
        *reinterpret_cast<float2*>(o + (r0 * a.H + h) * 128 + col) = make_float2(oacc[j][0] * i0, oacc[j][1] * i0);
        *reinterpret_cast<float2*>(o + (r1 * a.H + h) * 128 + col) = make_float2(oacc[j][2] * i1, oacc[j][3] * i1);
      } else {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);
        *reinterpret_cast<uint32_t*>(o + (r0 * a.H + h) * 128 + col) = pack_bf16(oacc[j][0] * i0, oacc[j][1] * i0);
        *reinterpret_cast<uint32_t*>(o + (r1 * a.H + h) * 128 + col) = pack_bf16(oacc[j][2] * i1, oacc[j][3] * i1);
      }
    }
  }
  if (bad && a.err) atomicExch(a.err, int(WAM_ERR_TIMEOUT));
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t s) {
  if (a.fl.n_items == 0) return cudaSuccess;
  PrefillMaps maps;
  const int qtok = (a.f_end - a.f_begin) * a.T, N = a.F * a.T;
  if (!make_tmap_bf16(&maps.q, a.q, a.B, qtok, a.H, kBM) ||
      !make_tmap_bf16(&maps.kn, a.k_new, a.B, qtok, a.H, kBN) ||
      !make_tmap_bf16(&maps.vn, a.v_new, a.B, qtok, a.H, kBN))
    return cudaErrorInvalidValue;
  if (a.f_begin > 0) {
    if (!make_tmap_bf16(&maps.kc, a.k_cache, a.B, N, a.H, kBN) ||
        !make_tmap_bf16(&maps.vc, a.v_cache, a.B, N, a.H, kBN))
      return cudaErrorInvalidValue;
  } else {
    maps.kc = maps.kn, maps.vc = maps.vn;
  }
  static unsigned configured = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 32) return cudaErrorInvalidDevice;
  if (!(configured & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(prefill_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured |= 1u << dev;
  }
  const int64_t grid = int64_t(a.fl.n_items) * (a.T / kBM) * a.H;
  prefill_mma_kernel<<<unsigned(grid), kThreads, kSmemBytes, s>>>(a, maps);
  return cudaGetLastError();
}

}  // namespace wam
