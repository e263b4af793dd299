// Asymmetric action attention on the tensor cores (bf16, D = 128, T % 64 == 0, n_act <= 32).
//
// 32 action queries read the fused video cache of one interaction layer plus their own K/V
// ("Fast-WAM 精读" SECTION 07; Long-WAM Summary §4.2).  The read is HBM-bound: per key it
// moves 512 B (K and V, bf16) and does 32 x 4 x 128 FLOP, 32 FLOP/B, above what the fp32
// pipes can issue at full HBM bandwidth, so the contractions run on mma.sync tensor-core
// tiles (M = 32 queries) while the loads stream through TMA: Q K^T on bf16 tiles, P V on tf32
// tiles (the fused cache is already rounded to bf16 once, so P is kept at 10 mantissa bits
// to leave the error budget to the storage rounding).
//
// Grid = (C splits, H, B), launched as clusters of C CTAs.  Split c of (b, h) reads a
// contiguous run of 64-key tiles of the episode's valid frames; split 0 also reads the
// action tile.  Each CTA keeps an fp32 online-softmax partial per key half; the 2C partials
// of a (b, h) are merged through distributed shared memory, so no workspace is needed.
//
// Warp roles: warps 0-3 consume (warp w: query rows 16*(w&1).., keys 32*(w>>1).. of each
// tile), warp 4 lane 0 issues the TMA loads.  3-stage K/V ring with full/empty mbarriers.
#include <cooperative_groups.h>

#include "launch.h"

namespace cg = cooperative_groups;

namespace wam {
namespace {

constexpr int kBN = 64;          // keys per tile
constexpr int kStages = 3;
constexpr int kConsumers = 4;    // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kQBytes = 32 * 128 * 2;
constexpr int kTileBytes = kBN * 128 * 2;   // one of K or V
constexpr int kOStride = 132;               // fp32 row stride of the merge buffers
constexpr int kSmemBytes = 1024 + kQBytes + kStages * 2 * kTileBytes + 256;

struct ActionMaps {
  CUtensorMap q, ka, va, fk, fv;
};

struct SmemLayout {
  uint8_t* q;
  uint8_t* k[kStages];
  uint8_t* v[kStages];
  uint64_t* full;
  uint64_t* empty;
  uint64_t* qbar;
  // merge area (aliases the K/V ring once every load has landed)
  float* obuf;    // [2][32][kOStride]
  float* mbuf;    // [2][32]
  float* lbuf;    // [2][32]
  float* fbuf;    // [32][2 * 16]
};

__device__ __forceinline__ SmemLayout carve(uint8_t* raw) {
  SmemLayout s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.q = base;
  uint8_t* p = base + kQBytes;
  for (int i = 0; i < kStages; ++i) {
    s.k[i] = p;
    s.v[i] = p + kTileBytes;
    p += 2 * kTileBytes;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(p);
  s.full = bars;
  s.empty = bars + kStages;
  s.qbar = bars + 2 * kStages;
  float* m = reinterpret_cast<float*>(base + kQBytes);
  s.obuf = m;
  s.mbuf = m + 2 * 32 * kOStride;
  s.lbuf = s.mbuf + 64;
  s.fbuf = s.lbuf + 64;
  return s;
}

__global__ void __launch_bounds__(kThreads, 2)
action_tc_kernel(const __grid_constant__ ActionArgs a, const __grid_constant__ ActionMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  SmemLayout sm = carve(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int split = int(cluster.block_rank());
  const int C = a.splits, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tiles of this split: [t0, t1) of the episode's valid video tiles, plus the action tile
  const int tiles_per_frame = a.T / kBN;
  const int nvt = a.with_video ? int(a.fl.nvalid[b]) * tiles_per_frame : 0;
  const int per = (nvt + C - 1) / C;
  const int t0 = min(nvt, split * per), t1 = min(nvt, t0 + per);
  const int has_act = split == 0 ? 1 : 0;
  const int n_tiles = (t1 - t0) + has_act;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kConsumers);
    }
    mbar_init(sm.qbar, 1);
    fence_barrier_init();
  }
  __syncthreads();

  bool bad = false;
  if (warp == kConsumers) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&maps.q);
      mbar_arrive_expect_tx(sm.qbar, kQBytes);
      tma_load_4d(sm.q, &maps.q, sm.qbar, 0, h, 0, b);
      tma_load_4d(sm.q + kQBytes / 2, &maps.q, sm.qbar, 64, h, 0, b);
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int st = i % kStages;
        if (i >= kStages && !mbar_wait(&sm.empty[st], ((i / kStages) - 1) & 1)) { bad = true; break; }
        mbar_arrive_expect_tx(&sm.full[st], 2 * kTileBytes);
        const CUtensorMap *mk, *mv;
        int tok;
        if (has_act && i == 0) {
          mk = &maps.ka, mv = &maps.va, tok = 0;
        } else {
          const int t = t0 + i - has_act;
          mk = &maps.fk, mv = &maps.fv;
          tok = int(a.fl.vlist[b * a.F + t / tiles_per_frame]) * a.T + (t % tiles_per_frame) * kBN;
        }
        tma_load_4d(sm.k[st], mk, &sm.full[st], 0, h, tok, b);
        tma_load_4d(sm.k[st] + kTileBytes / 2, mk, &sm.full[st], 64, h, tok, b);
        tma_load_4d(sm.v[st], mv, &sm.full[st], 0, h, tok, b);
        tma_load_4d(sm.v[st] + kTileBytes / 2, mv, &sm.full[st], 64, h, tok, b);
        issued = i + 1;
      }
      // Drain: every issued load must land before the ring is reused as merge space.
      for (int i = max(0, issued - kStages); i < issued; ++i)
        if (!mbar_wait(&sm.full[i % kStages], (i / kStages) & 1)) break;
      if (!mbar_wait(sm.qbar, 0)) bad = true;
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int qh = warp & 1, kh = warp >> 1;
    const int g = lane >> 2, t = lane & 3;
    float oacc[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    uint32_t qf[8][4];
    bad = !__all_sync(0xffffffffu, mbar_wait(sm.qbar, 0));  // warp-uniform before collectives
    if (!bad) {
      const uint32_t qbase = smem_u32(sm.q);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        ldsm_x4(qbase + swz128<32>(16 * qh + (lane & 15), 16 * kk + (lane >> 4) * 8), qf[kk][0],
                qf[kk][1], qf[kk][2], qf[kk][3]);
    }
    const float c = a.scale_log2;
    for (int i = 0; i < n_tiles && !bad; ++i) {
      const int st = i % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[st], (i / kStages) & 1))) { bad = true; break; }
      const uint32_t kb = smem_u32(sm.k[st]), vb = smem_u32(sm.v[st]);
      // S = Q K^T for this warp's 16 rows x 32 keys
      float s[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + swz128<kBN>(32 * kh + 16 * p + (lane & 7) + (lane >> 4) * 8,
                                   16 * kk + ((lane >> 3) & 1) * 8),
                  b0, b1, b2, b3);
          mma_bf16(s[2 * p], qf[kk], b0, b1);
          mma_bf16(s[2 * p + 1], qf[kk], b2, b3);
        }
      }
      if (has_act && i == 0) {  // action tile: keys >= n_act are the zero-filled tail
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int key = 32 * kh + 8 * j + 2 * t;
          if (key >= a.n_act) s[j][0] = s[j][2] = -INFINITY;
          if (key + 1 >= a.n_act) s[j][1] = s[j][3] = -INFINITY;
        }
      }
      // online softmax (rows g and g + 8), quad shuffles for the row reductions
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
        mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0 * c), mn1 = fmaxf(m1, mx1 * c);
      const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = exp2f(m0 - mu0), al1 = exp2f(m1 - mu1);
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s[j][0] = exp2f(fmaf(s[j][0], c, -mu0));
        s[j][1] = exp2f(fmaf(s[j][1], c, -mu0));
        s[j][2] = exp2f(fmaf(s[j][2], c, -mu1));
        s[j][3] = exp2f(fmaf(s[j][3], c, -mu1));
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
      // O += P V over this warp's 32 keys on tf32 tiles (m16n8k8): P keeps 10 mantissa bits
      // instead of bf16's 7, and V widens from bf16 to tf32 exactly.  Within each 8-key group
      // j the contraction index is permuted (logical k = t <-> key 8j + 2t, k = t + 4 <->
      // key 8j + 2t + 1), which makes the S accumulators the A fragment and the two keys an
      // ldmatrix.trans register holds the B fragment, with no data movement.
      uint32_t pt[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        pt[j][0] = to_tf32(s[j][0]);  // row g,     key 8j + 2t
        pt[j][1] = to_tf32(s[j][2]);  // row g + 8, key 8j + 2t
        pt[j][2] = to_tf32(s[j][1]);  // row g,     key 8j + 2t + 1
        pt[j][3] = to_tf32(s[j][3]);  // row g + 8, key 8j + 2t + 1
      }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int j0 = 2 * kk, j1 = 2 * kk + 1;  // 8-key groups of this 16-key step
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4_t(vb + swz128<kBN>(32 * kh + 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8,
                                     16 * p + (lane >> 4) * 8),
                    r0, r1, r2, r3);
          mma_tf32(oacc[2 * p], pt[j0][0], pt[j0][1], pt[j0][2], pt[j0][3], bf16_lo_bits(r0), bf16_hi_bits(r0));
          mma_tf32(oacc[2 * p], pt[j1][0], pt[j1][1], pt[j1][2], pt[j1][3], bf16_lo_bits(r1), bf16_hi_bits(r1));
          mma_tf32(oacc[2 * p + 1], pt[j0][0], pt[j0][1], pt[j0][2], pt[j0][3], bf16_lo_bits(r2), bf16_hi_bits(r2));
          mma_tf32(oacc[2 * p + 1], pt[j1][0], pt[j1][1], pt[j1][2], pt[j1][3], bf16_lo_bits(r3), bf16_hi_bits(r3));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[st]);
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    // The ring becomes merge space once every consumer left the loop and the producer
    // drained its loads: named barrier 1 over all threads of the CTA.
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads));
    // partial of this warp -> obuf[kh]
    float* ob = sm.obuf + kh * 32 * kOStride;
    const int r0 = 16 * qh + g, r1 = r0 + 8;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      *reinterpret_cast<float2*>(ob + r0 * kOStride + 8 * j + 2 * t) = make_float2(oacc[j][0], oacc[j][1]);
      *reinterpret_cast<float2*>(ob + r1 * kOStride + 8 * j + 2 * t) = make_float2(oacc[j][2], oacc[j][3]);
    }
    if (t == 0) {
      sm.mbuf[kh * 32 + r0] = m0, sm.mbuf[kh * 32 + r1] = m1;
      sm.lbuf[kh * 32 + r0] = l0, sm.lbuf[kh * 32 + r1] = l1;
    }
  }
  if (warp == kConsumers) {
    __syncwarp();  // lane 0 ran the producer loop alone
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads));
  }
  if (bad && a.err) atomicExch(a.err, int(WAM_ERR_TIMEOUT));

  // ------------------------------------------------------------------ cluster merge
  __syncwarp();
  cluster.sync();
  const int P = 2 * C;  // partials per (b, h)
  if (threadIdx.x < 32) {
    const int row = threadIdx.x;
    float mv[32], M = -INFINITY;
    for (int p = 0; p < P; ++p) {
      const float* rm = cluster.map_shared_rank(sm.mbuf, p >> 1);
      mv[p] = rm[(p & 1) * 32 + row];
      M = fmaxf(M, mv[p]);
    }
    if (M == -INFINITY) M = 0.f;
    float L = 0.f;
    for (int p = 0; p < P; ++p) {
      const float* rl = cluster.map_shared_rank(sm.lbuf, p >> 1);
      mv[p] = exp2f(mv[p] - M);
      L = fmaf(rl[(p & 1) * 32 + row], mv[p], L);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int p = 0; p < P; ++p) sm.fbuf[row * 32 + p] = mv[p] * inv;
  }
  __syncthreads();
  const int rows_per = 32 / C;
  const int rb = split * rows_per;
  if (threadIdx.x < 128) {
    const int col = (threadIdx.x & 31) * 4;
    for (int row = rb + (threadIdx.x >> 5); row < rb + rows_per; row += 4) {
      if (row >= a.n_act) break;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int p = 0; p < P; ++p) {
        const float* ro = cluster.map_shared_rank(sm.obuf, p >> 1);
        const float4 x = *reinterpret_cast<const float4*>(ro + (p & 1) * 32 * kOStride + row * kOStride + col);
        const float f = sm.fbuf[row * 32 + p];
        acc.x = fmaf(f, x.x, acc.x), acc.y = fmaf(f, x.y, acc.y);
        acc.z = fmaf(f, x.z, acc.z), acc.w = fmaf(f, x.w, acc.w);
      }
      const int64_t off = ((int64_t(b) * a.n_act + row) * a.H + h) * 128 + col;
      if (a.o_f32) {
        *reinterpret_cast<float4*>(static_cast<float*>(a.o) + off) = acc;
      } else {
        uint2 u;
        u.x = pack_bf16(acc.x, acc.y);
        u.y = pack_bf16(acc.z, acc.w);
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.o) + off) = u;
      }
    }
  }
  cluster.sync();  // keep this CTA's shared memory alive until every peer has read it
}

int pick_splits(const ActionArgs& a) {
  if (!a.with_video) return 1;
  int maxv = 0;
  for (int b = 0; b < a.B; ++b) maxv = maxv > a.fl.nvalid[b] ? maxv : a.fl.nvalid[b];
  const int tiles = maxv * (a.T / kBN);
  const int target = 2 * 148;  // two resident CTAs per SM
  int C = 1;
  while (C < 16 && a.B * a.H * C < target && tiles / (2 * C) >= 4) C *= 2;
  return C;
}

}  // namespace

cudaError_t launch_action_tc(const ActionArgs& args, cudaStream_t s) {
  ActionArgs a = args;
  a.splits = pick_splits(a);
  ActionMaps maps;
  const int N = a.F * a.T;
  if (!make_tmap_bf16(&maps.q, a.qa, a.B, a.n_act, a.H, 32) ||
      !make_tmap_bf16(&maps.ka, a.ka, a.B, a.n_act, a.H, kBN) ||
      !make_tmap_bf16(&maps.va, a.va, a.B, a.n_act, a.H, kBN))
    return cudaErrorInvalidValue;
  if (a.with_video) {
    if (!make_tmap_bf16(&maps.fk, a.fk, a.B, N, a.H, kBN) ||
        !make_tmap_bf16(&maps.fv, a.fv, a.B, N, a.H, kBN))
      return cudaErrorInvalidValue;
  } else {
    maps.fk = maps.ka, maps.fv = maps.va;
  }
  static unsigned configured = 0;  // one bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 32) return cudaErrorInvalidDevice;
  if (!(configured & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(action_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(action_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    configured |= 1u << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.splits, a.H, a.B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, action_tc_kernel, a, maps);
}

}  // namespace wam
