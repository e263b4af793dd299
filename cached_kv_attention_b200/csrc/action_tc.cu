// Asymmetric action attention: 32 action queries read the fused video cache of one
// interaction layer plus their own K/V ("Fast-WAM 精读" SECTION 07; Long-WAM Summary §4.2).
// The read is HBM-bound: per key it moves 512 B (K and V, bf16) for 32 x 4 x 128 FLOP.
// Four kernels (bf16, D = 128, n_act <= 32):
//   action_umma_kernel  T % 128 == 0: tcgen05 tensor cores, one thread-block cluster per
//                       (episode, head), partials merged in distributed shared memory (below).
//   action_nvfp4_kernel the same read over an NVFP4 fused pair (wam_action_attn_nvfp4): every
//                       head cut at the same tile boundaries, one part per CTA, partials merged
//                       through the workspace (below).
//   action_tc_kernel    T % 64 == 0 otherwise: mma.sync tiles (M = 32 queries), Q K^T on bf16
//                       and P V on tf32 (P keeps 10 mantissa bits; the fused cache is already
//                       rounded to bf16 once).  Persistent and balanced: the call's tiles (per
//                       (episode b, head h) one action tile, the n_act action keys zero-padded
//                       to 64 and masked, then the 64-key tiles of b's valid frames) are cut
//                       into P equal runs, one per CTA (P = SM count).  A CTA keeps one
//                       online-softmax state per (b, h) run it touches; a (b, h) contained in
//                       one CTA writes O directly, otherwise each CTA writes its partial
//                       (O, m, l) into the workspace and the last to arrive (atomic ticket)
//                       merges them by their log-sum-exp and resets the ticket.  Warps 0-7
//                       consume (warp w: query rows 16 (w & 1) .., keys (w >> 1) * 16 .. of
//                       each tile), warp 8 lane 0 issues TMA loads into a 4-stage ring and a
//                       2-slot Q buffer.
//   action_self_kernel  layers outside the interaction set (action keys only).
#include <cuda_fp16.h>

#include <mutex>

#include "launch.h"
#include "tcgen05.cuh"

namespace wam {
namespace {

constexpr int kRingBytes = 128 * 1024;    // K/V ring: 2 stages of 128 keys or 4 of 64
constexpr int kConsumers = 8;
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kQBytes = 32 * 128 * 2;
constexpr int kOStride = 132;               // fp32 row stride of the merge buffers
constexpr int kSlotFloats = 32 * 128 + 64;  // one workspace partial: O [32][128], m [32], l [32]
constexpr int kMergeBytes = 4 * 32 * kOStride * 4 + 2 * 4 * 32 * 4;
constexpr int kSmemBytes = 1024 + 2 * kQBytes + kRingBytes + kMergeBytes + 256;
constexpr int kMaxStages = 4;
constexpr float kLazyLog2 = 8.f;  // headroom of a row's softmax reference (log2 units)

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct ActionMaps {
  CUtensorMap q, ka, va, fk, fv;
};

struct Bars {
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t qfull[2], qempty[2];
  int last;  // merge flag of the current run
};

template <int kBN>
__device__ __forceinline__ int tiles_of(const ActionArgs& a, int b) {
  return 1 + (a.with_video ? int(a.fl.nvalid[b]) * (a.T / kBN) : 0);
}

// Walks the call's tile sequence: (b, h, t) of global tile g, nb tiles per (b, h).
template <int kBN>
struct TileWalk {
  int b, h, t, nb;
  __device__ __forceinline__ void init(const ActionArgs& a, int g) {
    b = 0;
    for (;;) {
      nb = tiles_of<kBN>(a, b);
      if (g < a.H * nb || b == a.B - 1) break;
      g -= a.H * nb;
      ++b;
    }
    h = g / nb;
    t = g % nb;
  }
  __device__ __forceinline__ void init_at(const ActionArgs& a, int b_, int h_, int t_) {
    b = b_, h = h_, t = t_, nb = tiles_of<kBN>(a, b_);
  }
  __device__ __forceinline__ void next(const ActionArgs& a) {
    if (++t < nb) return;
    t = 0;
    if (++h < a.H) return;
    h = 0;
    if (++b < a.B) nb = tiles_of<kBN>(a, b);
  }
};

template <int kBN>
__device__ __forceinline__ int first_tile_of(const ActionArgs& a, int b, int h) {
  int g = 0;
  for (int e = 0; e < b; ++e) g += a.H * tiles_of<kBN>(a, e);
  return g + h * tiles_of<kBN>(a, b);
}

// First and last CTA whose run touches tiles [s, e) when CTA i runs [iG/P, (i+1)G/P).
__device__ __forceinline__ int cta_of_start(int s, int G, int P) {
  return int((int64_t(s + 1) * P + G - 1) / G) - 1;
}
__device__ __forceinline__ int cta_of_end(int e, int G, int P) {
  return int((int64_t(e) * P + G - 1) / G) - 1;
}

__device__ __forceinline__ void store_out(const ActionArgs& a, int b, int h, int row, int col,
                                          const float* v /*16*/) {
  const int64_t off = ((int64_t(b) * a.n_act + row) * a.H + h) * 128 + col;
  if (a.o_f32) {
    float4* d = reinterpret_cast<float4*>(static_cast<float*>(a.o) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else {
    uint4* d = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + off);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint4 u;
      u.x = pack_bf16(v[8 * i], v[8 * i + 1]), u.y = pack_bf16(v[8 * i + 2], v[8 * i + 3]);
      u.z = pack_bf16(v[8 * i + 4], v[8 * i + 5]), u.w = pack_bf16(v[8 * i + 6], v[8 * i + 7]);
      d[i] = u;
    }
  }
}

// kBN keys per tile (64 or 128); each consumer warp handles kBN / 4 keys of a tile.
template <int kBN>
__global__ void __launch_bounds__(kThreads, 1)
action_tc_kernel(const __grid_constant__ ActionArgs a, const __grid_constant__ ActionMaps maps) {
  constexpr int kTileBytes = kBN * 128 * 2;  // one of K or V
  constexpr int kStages = kRingBytes / (2 * kTileBytes);
  constexpr int kWK = kBN / 4;               // keys per warp per tile
  constexpr int kNT = kWK / 8;               // 8-key groups per warp per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  uint8_t* sq[2] = {base, base + kQBytes};
  uint8_t* sk[kStages];
  uint8_t* sv[kStages];
  for (int i = 0; i < kStages; ++i) {
    sk[i] = base + 2 * kQBytes + i * 2 * kTileBytes;
    sv[i] = sk[i] + kTileBytes;
  }
  float* obuf = reinterpret_cast<float*>(base + 2 * kQBytes + kStages * 2 * kTileBytes);  // [4][32][132]
  float* mbuf = obuf + 4 * 32 * kOStride;  // [4][32]
  float* lbuf = mbuf + 4 * 32;             // [4][32]
  Bars& bars = *reinterpret_cast<Bars*>(lbuf + 4 * 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g0 = int(int64_t(blockIdx.x) * a.G / a.P), g1 = int(int64_t(blockIdx.x + 1) * a.G / a.P);
  const int tpf = a.T / kBN;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars.full[i], 1);
      mbar_init(&bars.empty[i], kConsumers);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.qfull[i], 1);
      mbar_init(&bars.qempty[i], kConsumers);
    }
    fence_barrier_init();
  }
  __syncthreads();

  bool bad = false;
  if (warp == kConsumers) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      TileWalk<kBN> tw;
      tw.init(a, g0);
      int seg = 0, issued = 0;
      for (int g = g0; g < g1; ++g, tw.next(a)) {
        const int i = g - g0, st = i % kStages;
        if (g == g0 || tw.t == 0) {  // a new (b, h) run: its Q first
          const int qs = seg & 1;
          if (seg >= 2 && !mbar_wait(&bars.qempty[qs], ((seg >> 1) - 1) & 1)) { bad = true; break; }
          mbar_arrive_expect_tx(&bars.qfull[qs], kQBytes);
          tma_load_4d(sq[qs], &maps.q, &bars.qfull[qs], 0, tw.h, 0, tw.b);
          tma_load_4d(sq[qs] + kQBytes / 2, &maps.q, &bars.qfull[qs], 64, tw.h, 0, tw.b);
          ++seg;
        }
        if (i >= kStages && !mbar_wait(&bars.empty[st], ((i / kStages) - 1) & 1)) { bad = true; break; }
        mbar_arrive_expect_tx(&bars.full[st], 2 * kTileBytes);
        const CUtensorMap *mk, *mv;
        int tok;
        if (tw.t == 0) {
          mk = &maps.ka, mv = &maps.va, tok = 0;
        } else {
          const int vt = tw.t - 1;
          mk = &maps.fk, mv = &maps.fv;
          tok = int(a.fl.vlist[tw.b * a.F + vt / tpf]) * a.T + (vt % tpf) * kBN;
        }
        tma_load_4d(sk[st], mk, &bars.full[st], 0, tw.h, tok, tw.b);
        tma_load_4d(sk[st] + kTileBytes / 2, mk, &bars.full[st], 64, tw.h, tok, tw.b);
        tma_load_4d(sv[st], mv, &bars.full[st], 0, tw.h, tok, tw.b);
        tma_load_4d(sv[st] + kTileBytes / 2, mv, &bars.full[st], 64, tw.h, tok, tw.b);
        issued = i + 1;
      }
      // Drain the loads still in flight (only after a failed wait can any be outstanding).
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_wait(&bars.full[i % kStages], (i / kStages) & 1);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers
    // Every wait in front of a warp-collective (ldmatrix, mma.sync) is voted across the warp;
    // after a failed wait a warp keeps walking its tiles and runs without doing work, and it
    // still arrives on every barrier and ticket, so peers and later calls are not stranded.
    const unsigned FULL = 0xffffffffu;
    const int qh = warp & 1, kq = warp >> 1;
    const int g = lane >> 2, t4 = lane & 3;
    const int tid = threadIdx.x;  // 0..255
    const float c = a.scale_log2;
    TileWalk<kBN> tw;
    tw.init(a, g0);
    int seg = 0;
    int gi = g0;
    while (gi < g1) {
      // ---- one (b, h) run [gi, ge) of this CTA
      const int b = tw.b, h = tw.h;
      const int ge = min(g1, gi + (tw.nb - tw.t));
      const int s_bh = first_tile_of<kBN>(a, b, h), e_bh = s_bh + tw.nb;
      const int qs = seg & 1;
      uint32_t qf[8][4];
      bad = bad || !__all_sync(FULL, mbar_wait(&bars.qfull[qs], (seg >> 1) & 1));
      if (!bad) {
        const uint32_t qbase = smem_u32(sq[qs]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ldsm_x4(qbase + swz128<32>(16 * qh + (lane & 15), 16 * kk + (lane >> 4) * 8), qf[kk][0],
                  qf[kk][1], qf[kk][2], qf[kk][3]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.qempty[qs]);
      float oacc[16][4];
#pragma unroll
      for (int j = 0; j < 16; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      for (; gi < ge; ++gi, tw.next(a)) {
        const int i = gi - g0, st = i % kStages;
        if (!bad && !__all_sync(FULL, mbar_wait(&bars.full[st], (i / kStages) & 1))) bad = true;
        if (!bad) {
          const uint32_t kb = smem_u32(sk[st]), vb = smem_u32(sv[st]);
          // S = Q K^T: this warp's 16 rows x kWK keys (kNT independent 8-key accumulators)
          const int kbase = kWK * kq;
          float s[kNT][4];
#pragma unroll
          for (int j = 0; j < kNT; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
            for (int p = 0; p < kNT / 2; ++p) {
              uint32_t b0, b1, b2, b3;
              ldsm_x4(kb + swz128<kBN>(kbase + 16 * p + (lane & 7) + (lane >> 4) * 8,
                                       16 * kk + ((lane >> 3) & 1) * 8),
                      b0, b1, b2, b3);
              mma_bf16(s[2 * p], qf[kk], b0, b1);
              mma_bf16(s[2 * p + 1], qf[kk], b2, b3);
            }
          }
          if (tw.t == 0) {  // action tile: keys >= n_act are the zero-filled tail
#pragma unroll
            for (int j = 0; j < kNT; ++j) {
              const int key = kbase + 8 * j + 2 * t4;
              if (key >= a.n_act) s[j][0] = s[j][2] = -INFINITY;
              if (key + 1 >= a.n_act) s[j][1] = s[j][3] = -INFINITY;
            }
          }
          // online softmax (rows g and g + 8), quad shuffles for the row reductions
          float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
          for (int j = 0; j < kNT; ++j) {
            mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
            mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
          }
          mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 1));
          mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 2));
          mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 1));
          mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 2));
          // The reference max of a row only moves when the tile's max exceeds it by more than
          // 2^8 (p = 2^(s c - m) then stays below 2^8), so the accumulators are rarely rescaled;
          // the rescale runs only when some row of the warp needs it.
          const float c0 = mx0 * c, c1 = mx1 * c;
          const float mn0 = c0 > m0 + kLazyLog2 ? c0 : m0, mn1 = c1 > m1 + kLazyLog2 ? c1 : m1;
          const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
          float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
          for (int j = 0; j < kNT; ++j) {
            s[j][0] = ex2(fmaf(s[j][0], c, -mu0));
            s[j][1] = ex2(fmaf(s[j][1], c, -mu0));
            s[j][2] = ex2(fmaf(s[j][2], c, -mu1));
            s[j][3] = ex2(fmaf(s[j][3], c, -mu1));
            rs0 += s[j][0] + s[j][1];
            rs1 += s[j][2] + s[j][3];
          }
          if (__any_sync(FULL, mn0 != m0 || mn1 != m1)) {
            const float al0 = ex2(m0 - mu0), al1 = ex2(m1 - mu1);
            l0 *= al0, l1 *= al1;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              oacc[j][0] *= al0, oacc[j][1] *= al0, oacc[j][2] *= al1, oacc[j][3] *= al1;
            }
          }
          l0 += rs0, l1 += rs1;
          m0 = mn0, m1 = mn1;
          // O += P V over this warp's keys on tf32 tiles (m16n8k8).  Within each 8-key group
          // j the contraction index is permuted (k = t <-> key 8j + 2t, k = t + 4 <-> 8j + 2t + 1)
          // so the S accumulators are the A fragment and the two keys of an ldmatrix.trans
          // register are the B fragment, with no data movement.
          uint32_t pt[kNT][4];
#pragma unroll
          for (int j = 0; j < kNT; ++j) {
            pt[j][0] = to_tf32(s[j][0]);
            pt[j][1] = to_tf32(s[j][2]);
            pt[j][2] = to_tf32(s[j][1]);
            pt[j][3] = to_tf32(s[j][3]);
          }
#pragma unroll
          for (int kb16 = 0; kb16 < kNT / 2; ++kb16) {
            const int j0 = 2 * kb16, j1 = 2 * kb16 + 1;
#pragma unroll
            for (int p = 0; p < 8; ++p) {
              uint32_t r0, r1, r2, r3;
              ldsm_x4_t(vb + swz128<kBN>(kbase + 16 * kb16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                                         16 * p + (lane >> 4) * 8),
                        r0, r1, r2, r3);
              mma_tf32(oacc[2 * p], pt[j0][0], pt[j0][1], pt[j0][2], pt[j0][3], bf16_lo_bits(r0), bf16_hi_bits(r0));
              mma_tf32(oacc[2 * p], pt[j1][0], pt[j1][1], pt[j1][2], pt[j1][3], bf16_lo_bits(r1), bf16_hi_bits(r1));
              mma_tf32(oacc[2 * p + 1], pt[j0][0], pt[j0][1], pt[j0][2], pt[j0][3], bf16_lo_bits(r2), bf16_hi_bits(r2));
              mma_tf32(oacc[2 * p + 1], pt[j1][0], pt[j1][1], pt[j1][2], pt[j1][3], bf16_lo_bits(r3), bf16_hi_bits(r3));
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.empty[st]);
      }
      ++seg;
      // ---- run done: the four key quarters of each query half -> one partial for 32 rows
      l0 += __shfl_xor_sync(FULL, l0, 1);
      l0 += __shfl_xor_sync(FULL, l0, 2);
      l1 += __shfl_xor_sync(FULL, l1, 1);
      l1 += __shfl_xor_sync(FULL, l1, 2);
      {
        float* ob = obuf + kq * 32 * kOStride;
        const int r0 = 16 * qh + g, r1 = r0 + 8;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          *reinterpret_cast<float2*>(ob + r0 * kOStride + 8 * j + 2 * t4) = make_float2(oacc[j][0], oacc[j][1]);
          *reinterpret_cast<float2*>(ob + r1 * kOStride + 8 * j + 2 * t4) = make_float2(oacc[j][2], oacc[j][3]);
        }
        if (t4 == 0) {
          mbuf[kq * 32 + r0] = m0, mbuf[kq * 32 + r1] = m1;
          lbuf[kq * 32 + r0] = l0, lbuf[kq * 32 + r1] = l1;
        }
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      // thread -> (row, 16 columns) of the 32 x 128 partial
      const int row = tid >> 3, col = (tid & 7) * 16;
      float M = -INFINITY;
#pragma unroll
      for (int k = 0; k < 4; ++k) M = fmaxf(M, mbuf[k * 32 + row]);
      const float Mu = M == -INFINITY ? 0.f : M;
      float fk[4], L = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        fk[k] = exp2f(mbuf[k * 32 + row] - Mu);
        L = fmaf(lbuf[k * 32 + row], fk[k], L);
      }
      float ov[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) ov[i] = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 x = *reinterpret_cast<const float4*>(obuf + (k * 32 + row) * kOStride + col + i);
          ov[i] = fmaf(fk[k], x.x, ov[i]), ov[i + 1] = fmaf(fk[k], x.y, ov[i + 1]);
          ov[i + 2] = fmaf(fk[k], x.z, ov[i + 2]), ov[i + 3] = fmaf(fk[k], x.w, ov[i + 3]);
        }
      const int bh = b * a.H + h;
      if (s_bh >= g0 && e_bh <= g1) {
        // this CTA holds the whole (b, h): write O directly
        if (row < a.n_act) {
          const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) ov[i] *= inv;
          store_out(a, b, h, row, col, ov);
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");  // merge buffers reused by the next run
      } else {
        // partial -> workspace slot (b, h, this CTA's rank among the CTAs touching (b, h))
        const int i_lo = cta_of_start(s_bh, a.G, a.P), n_parts = cta_of_end(e_bh, a.G, a.P) - i_lo + 1;
        float* slot = a.ws_part + (int64_t(bh) * a.max_parts + (int(blockIdx.x) - i_lo)) * kSlotFloats;
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          __stcg(reinterpret_cast<float4*>(slot + row * 128 + col + i), make_float4(ov[i], ov[i + 1], ov[i + 2], ov[i + 3]));
        if ((tid & 7) == 0) {
          __stcg(slot + 32 * 128 + row, M);
          __stcg(slot + 32 * 128 + 32 + row, L);
        }
        __threadfence();
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (tid == 0) bars.last = atomicAdd(a.ws_count + bh, 1) == n_parts - 1;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (bars.last) {
          // every partial of (b, h) is in the workspace: merge them by log-sum-exp
          __threadfence();
          const float* slots = a.ws_part + int64_t(bh) * a.max_parts * kSlotFloats;
          float Mt = -INFINITY;
          for (int k = 0; k < n_parts; ++k) Mt = fmaxf(Mt, __ldcg(slots + k * kSlotFloats + 32 * 128 + row));
          const float Mtu = Mt == -INFINITY ? 0.f : Mt;
          float Lt = 0.f, acc[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] = 0.f;
          // two partials per round, all their loads issued before any is used
          for (int k = 0; k < n_parts; k += 2) {
            const bool two = k + 1 < n_parts;
            const float* sa = slots + k * kSlotFloats;
            const float* sb = slots + (two ? k + 1 : k) * kSlotFloats;
            float4 xa[4], xb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              xa[i] = __ldcg(reinterpret_cast<const float4*>(sa + row * 128 + col + 4 * i));
              xb[i] = __ldcg(reinterpret_cast<const float4*>(sb + row * 128 + col + 4 * i));
            }
            const float ma = __ldcg(sa + 32 * 128 + row), la = __ldcg(sa + 32 * 128 + 32 + row);
            const float mb = __ldcg(sb + 32 * 128 + row), lb = __ldcg(sb + 32 * 128 + 32 + row);
            const float fa = exp2f(ma - Mtu), fb = two ? exp2f(mb - Mtu) : 0.f;
            Lt = fmaf(la, fa, fmaf(lb, fb, Lt));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc[4 * i] = fmaf(fa, xa[i].x, fmaf(fb, xb[i].x, acc[4 * i]));
              acc[4 * i + 1] = fmaf(fa, xa[i].y, fmaf(fb, xb[i].y, acc[4 * i + 1]));
              acc[4 * i + 2] = fmaf(fa, xa[i].z, fmaf(fb, xb[i].z, acc[4 * i + 2]));
              acc[4 * i + 3] = fmaf(fa, xa[i].w, fmaf(fb, xb[i].w, acc[4 * i + 3]));
            }
          }
          if (row < a.n_act) {
            const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] *= inv;
            store_out(a, b, h, row, col, acc);
          }
          if (tid == 0) a.ws_count[bh] = 0;  // ready for the next call
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
      }
    }
  }
  if (bad && a.err) atomicExch(a.err, int(WAM_ERR_TIMEOUT));
}

// ============================================================================================
// The same read on the sm_100 tensor cores, for 128-key tiles (T % 128 == 0).  It is written
// transposed so that the 128-row MMA is filled by keys rather than by the 32 queries:
//   S^T = K Q^T    M = 128 keys, N = 32 queries, K = D; both operands K-major in shared memory;
//   O^T += V^T P^T M = D = 128, N = 64 (32 query columns of P_hi, 32 of P_lo), K = 128 keys;
//                  V^T is the MN-major view of the V tile as TMA wrote it, P^T a tile of
//                  128-byte rows.
// S^T (two buffers) and O^T live in tensor memory.  Two softmax warpgroups: a thread takes one
// key (its TMEM lane) and the 16 queries of its group; each query keeps one reference max,
// shared by all threads, that moves (with O^T and the row sums rescaled) only when a tile
// exceeds it by more than 2^16, which one OR-reduction barrier per tile detects.
//
// Work split: one thread-block cluster of k <= 8 CTAs per (episode, head); CTA r of the
// cluster streams the r-th of k contiguous slices of the (episode, head)'s tiles (the action
// tile first, then the valid frames' tiles).  The k partials (O, m, l) meet in distributed
// shared memory and never leave the chip: CTA r owns query rows [r n_act / k, (r+1) n_act / k)
// and keeps a receive region for them, whose barrier it arms at start with every byte its
// peers will send.  After its loop a CTA sends each partial row to its owner with st.async
// stores counted on that barrier (its own rows are copied locally), then waits for its rows
// from every peer and merges them.  One one-way hop follows the slowest slice, and no CTA
// waits on another before leaving.
// Warps: 0 TMA producer, 1 TMEM owner and MMA issuer, 2-9 softmax (warp w: TMEM lane quarter
// w % 4, query group (w - 2) / 4).
namespace um {
constexpr int kKeys = 128;
constexpr int kTile = kKeys * 128 * 2;   // one of K or V: 32 KB
constexpr int kKStages = 3;            // K ring
constexpr int kVStages = 2;            // V ring (its tiles are needed one S^T later than K's)
constexpr int kQ = 32 * 128 * 2;         // 8 KB
constexpr int kP = kKeys * 128;          // P^T: 128 keys x (32 P_hi + 32 P_lo) bf16 = 16 KB
constexpr int kThreads = 10 * 32;       // producer, MMA issuer, 8 softmax warps
constexpr uint32_t kTmemCols = 128;      // S^T buffers at columns 0 and 32, O^T at 64
constexpr float kLazy = 16.f;            // reference headroom (log2 units): P <= 2^16
constexpr int kMaxSplit = 8;             // portable cluster size
struct Bars {
  uint64_t kfull[kKStages], kempty[kKStages], vfull[kVStages], vempty[kVStages];
  uint64_t qfull, sfull[2], sfree[2], pfull, pfree, ofull, done;
  uint32_t tmem_base;
  int abort;
  float red[8][16];  // per softmax warp: one value per query of its group
  // the merge over the cluster: completes once every peer's partial rows for this CTA have landed
  uint64_t rx_full;
  float part_m[32], part_l[32];  // this CTA's partial: reference max and row sum per query
  // where row q of this CTA's partial goes: the owner's rank, and the byte offsets of its O row
  // and of its (m, l) pair in the owner's receive region
  int row_owner[32], row_off[32], ml_off[32];
};
// Receive region of the merge: k slots (one per rank of the cluster) of this CTA's query rows,
// [slot][row][128 floats] then the (m, l) pairs [slot][row]; k x ceil(32 / k) x 520 bytes at most.
constexpr int kRx = 19 * 1024;
constexpr int rx_bytes(int k) { return k * ((32 + k - 1) / k) * 520; }
static_assert(rx_bytes(2) <= kRx && rx_bytes(3) <= kRx && rx_bytes(4) <= kRx && rx_bytes(5) <= kRx &&
                  rx_bytes(6) <= kRx && rx_bytes(7) <= kRx && rx_bytes(8) <= kRx,
              "receive region");
constexpr int kSmemBytes = 1024 + kQ + (kKStages + kVStages) * kTile + kP + kRx + int(sizeof(Bars)) + 64;
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(32 * 128 * 4 == kP, "the partial O [32][128] fp32 reuses the P^T buffer");

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < kWaitSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 31u && *abort) return false;
  }
  *abort = 1;
  return false;
}
// Named barrier 1 over the 128 softmax threads, and the same barrier with an OR-reduction.
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// The same over the 256 threads of two softmax warpgroups.
__device__ __forceinline__ void softmax8_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ bool softmax8_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n barrier.red.or.pred p, 1, 256, q;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(r)
      : "r"(uint32_t(v))
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool softmax_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n barrier.red.or.pred p, 1, 128, q;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(r)
      : "r"(uint32_t(v))
      : "memory");
  return r != 0;
}
// The address, in the cluster's shared window, of the byte at the offset of `local` in CTA
// `peer`'s shared memory.
__device__ __forceinline__ uint32_t peer_addr(const void* local, uint32_t peer) {
  uint32_t pa;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(pa) : "r"(smem_u32(local)), "r"(peer));
  return pa;
}
// Asynchronous stores into a peer's shared memory (cluster window addresses), each counted in
// bytes on the barrier at `bar` in that peer.
__device__ __forceinline__ void st_async4(uint32_t pa, float4 v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(pa),
               "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void st_async2(uint32_t pa, float x, float y, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(pa), "f"(x),
               "f"(y), "r"(bar)
               : "memory");
}
// A bounded wait on a local barrier that peers arrive on, acquiring their writes at cluster scope.
// It does not give up early when this CTA has aborted: peers may still write into this CTA's
// shared memory until they have arrived, and every peer runs the exchange whatever happened to
// it, so only the spin limit ends the wait (and then reports a timeout).
__device__ __forceinline__ bool wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < kWaitSpinLimit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  *abort = 1;
  return false;
}
// After the call lane q holds the max (or sum) over the warp's lanes of v[q]; v is clobbered.
template <bool kMax>
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool hi = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = hi ? v[i] : v[i + off];
      const float keep = hi ? v[i + off] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
}
// The same for 16 values: after the call lanes q and q + 16 hold the max (or sum) over the
// warp's lanes of v[q]; v is clobbered.
template <bool kMax>
__device__ __forceinline__ float reduce_scatter16(float (&v)[16], int lane) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float got = __shfl_xor_sync(0xffffffffu, v[i], 16);
    v[i] = kMax ? fmaxf(v[i], got) : v[i] + got;
  }
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) {
    const bool hi = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = hi ? v[i] : v[i + off];
      const float keep = hi ? v[i + off] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
}
}  // namespace um

__global__ void __launch_bounds__(um::kThreads, 1)
action_umma_kernel(const __grid_constant__ ActionArgs a, const __grid_constant__ ActionMaps maps) {
  using namespace um;
  // the tensor maps' descriptors first: fetching one takes about a microsecond, hidden behind
  // the set-up below (parameter space: the previous kernel on the stream cannot write it)
  if (threadIdx.x == 0) {
    prefetch_tmap(&maps.q), prefetch_tmap(&maps.ka), prefetch_tmap(&maps.va);
    prefetch_tmap(&maps.fk), prefetch_tmap(&maps.fv);
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  uint8_t* sQ = base;
  auto sK = [&](int st) { return base + kQ + st * kTile; };
  auto sV = [&](int st) { return base + kQ + (kKStages + st) * kTile; };
  uint8_t* sP = base + kQ + (kKStages + kVStages) * kTile;
  uint8_t* rx = sP + kP;  // receive region of the cluster merge (k > 1)
  um::Bars& bars = *reinterpret_cast<um::Bars*>(rx + kRx);
  volatile int* abort = &bars.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned FULL = 0xffffffffu;
  // this CTA's slice [t0, t1) of the tiles of (b, h): tile 0 the action keys, tile 1 + v the
  // v-th 128-key tile of b's valid frames
  const int k = a.ksplit;
  const int bh = int(blockIdx.x) / k, rank = int(blockIdx.x) % k;
  const int b = bh / a.H, h = bh % a.H;
  const int tpf = a.T / kKeys;
  const int nb = tiles_of<kKeys>(a, b);
  const int t0 = rank * nb / k, t1 = (rank + 1) * nb / k, n = t1 - t0;
  auto tile_src = [&](int i, bool is_v, const CUtensorMap*& mp, int& tok) {
    const int t = t0 + i;
    if (t == 0) {
      mp = is_v ? &maps.va : &maps.ka, tok = 0;
    } else {
      const int vt = t - 1;
      mp = is_v ? &maps.fv : &maps.fk;
      tok = int(a.fl.vlist[b * a.F + vt / tpf]) * a.T + (vt % tpf) * kKeys;
    }
  };
  auto load_kv = [&](int i) {  // K and V of the slice's tile i (i < both ring sizes)
    const CUtensorMap* mp;
    int tok;
    tile_src(i, false, mp, tok);
    mbar_arrive_expect_tx(&bars.kfull[i], kTile);
    tma_load_4d(sK(i), mp, &bars.kfull[i], 0, h, tok, b);
    tma_load_4d(sK(i) + kTile / 2, mp, &bars.kfull[i], 64, h, tok, b);
    tile_src(i, true, mp, tok);
    mbar_arrive_expect_tx(&bars.vfull[i], kTile);
    tma_load_4d(sV(i), mp, &bars.vfull[i], 0, h, tok, b);
    tma_load_4d(sV(i) + kTile / 2, mp, &bars.vfull[i], 64, h, tok, b);
  };
  const int n_pre = n < kVStages ? n : kVStages;  // kVStages <= kKStages
  uint32_t pre = 0;  // bit i: tile i requested before the dependency wait (thread 0)

  if (threadIdx.x == 0) {
    // the frame table's entries for the first tiles, fetched while the barriers are set up
    int warm = 0;
    for (int i = 0; i < n_pre; ++i) {
      const CUtensorMap* mp;
      int tok;
      tile_src(i, false, mp, tok);
      warm += tok;
    }
    asm volatile("" ::"r"(warm));
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bars.kfull[i], 1);
      mbar_init(&bars.kempty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&bars.vfull[i], 1);
      mbar_init(&bars.vempty[i], 1);
    }
    mbar_init(&bars.qfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.sfull[i], 1);
      mbar_init(&bars.sfree[i], 8);  // one arrival per softmax warp
    }
    mbar_init(&bars.pfull, 8);
    mbar_init(&bars.pfree, 1);
    mbar_init(&bars.ofull, 1);
    mbar_init(&bars.done, 1);
    bars.abort = 0;
    if (k > 1) {
      // armed now with every byte the k - 1 peers will send (their rows of this CTA's range),
      // before the cluster barrier below lets any of them send
      const int rows = (rank + 1) * a.n_act / k - rank * a.n_act / k;
      mbar_init(&bars.rx_full, 1);
      mbar_arrive_expect_tx(&bars.rx_full, uint32_t((k - 1) * rows * 520));
    }
    fence_barrier_init();
    // Up to here only this CTA's shared memory was touched: the previous kernel on the stream
    // may still be finishing (programmatic dependent launch).  With a.fused_ready the caller
    // guarantees that kernel does not write the fused pair, so the slice's first fused tiles
    // are requested now, by the thread that set up their barriers (the fence above makes them
    // visible to the copies); the action tile and Q wait for the dependency.
    if (a.fused_ready)
      for (int i = 0; i < n_pre; ++i)
        if (t0 + i != 0) load_kv(i), pre |= 1u << i;
  }
  if (warp == 1) {
    tc05::tmem_alloc(&bars.tmem_base, kTmemCols);
    tc05::tmem_relinquish();
  }
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  // every CTA of the cluster has initialised (and armed) its barriers once this phase completes
  // (the barrier-init fence above orders the initialisation; the receive barrier's byte count
  // may be armed after a peer's first bytes land); each thread waits on it before its first
  // access to a peer (the softmax warps) or before leaving
  if (k > 1) asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
  const uint32_t tmem = bars.tmem_base;
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // K and V stream through separate rings (3 and 2 stages): a K stage is refilled as soon as
    // its S^T MMA has completed, a V stage once its P V has.  The two sequences advance
    // independently.
    if (lane == 0 && n > 0) {
      mbar_arrive_expect_tx(&bars.qfull, kQ);
      tma_load_4d(sQ, &maps.q, &bars.qfull, 0, h, 0, b);
      tma_load_4d(sQ + kQ / 2, &maps.q, &bars.qfull, 64, h, 0, b);
      for (int i = 0; i < n_pre; ++i)  // the first stages: those not requested above
        if (!((pre >> i) & 1u)) load_kv(i);
      int nk = n_pre, nv = n_pre;
      for (uint32_t it = 0; (nk < n || nv < n) && it < kWaitSpinLimit; ++it) {
        if ((it & 31u) == 31u && *abort) break;
        const int nk0 = nk, nv0 = nv;
        if (nk < n && (nk < kKStages || mbar_test_wait(&bars.kempty[nk % kKStages], ((nk / kKStages) - 1) & 1))) {
          const int st = nk % kKStages;
          const CUtensorMap* mp;
          int tok;
          tile_src(nk, false, mp, tok);
          mbar_arrive_expect_tx(&bars.kfull[st], kTile);
          tma_load_4d(sK(st), mp, &bars.kfull[st], 0, h, tok, b);
          tma_load_4d(sK(st) + kTile / 2, mp, &bars.kfull[st], 64, h, tok, b);
          ++nk;
        }
        if (nv < n && (nv < kVStages || mbar_test_wait(&bars.vempty[nv % kVStages], ((nv / kVStages) - 1) & 1))) {
          const int st = nv % kVStages;
          const CUtensorMap* mp;
          int tok;
          tile_src(nv, true, mp, tok);
          mbar_arrive_expect_tx(&bars.vfull[st], kTile);
          tma_load_4d(sV(st), mp, &bars.vfull[st], 0, h, tok, b);
          tma_load_4d(sV(st) + kTile / 2, mp, &bars.vfull[st], 64, h, tok, b);
          ++nv;
        }
        if (nk == nk0 && nv == nv0) poll_pause();
      }
      if (nk < n || nv < n) *abort = 1;
      // Loads still in flight land before the CTA leaves (only after an abort can any be).
      for (int i = (nk > kKStages ? nk - kKStages : 0); i < nk; ++i) mbar_wait(&bars.kfull[i % kKStages], (i / kKStages) & 1);
      for (int i = (nv > kVStages ? nv - kVStages : 0); i < nv; ++i) mbar_wait(&bars.vfull[i % kVStages], (i / kVStages) & 1);
      mbar_wait(&bars.qfull, 0);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // S^T of up to two tiles ahead is issued as soon as its K tile has landed and its tensor-
    // memory buffer has been read, while P V of the current tile waits for its P: the softmax
    // of tile i + 1 never waits for P V of tile i.
    if (lane == 0) {
      const uint32_t idS = tc05::idesc_bf16_f32(128, 32, false, false);
      const uint32_t idO = tc05::idesc_bf16_f32(128, 64, true, true);
      auto s_ready = [&](int j) {
        return mbar_test_wait(&bars.kfull[j % kKStages], (j / kKStages) & 1) &&
               (j > 0 || mbar_test_wait(&bars.qfull, 0)) &&
               (j < 2 || mbar_test_wait(&bars.sfree[j & 1], ((j >> 1) - 1) & 1));
      };
      auto issue_S = [&](int j) {
        const int st = j % kKStages;
        tc05::fence_after_sync();
        const uint32_t k_s = smem_u32(sK(st)), q_s = smem_u32(sQ);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc05::mma_ss(tmem + 32 * (j & 1),
                       tc05::smem_desc_sw128(k_s + (kk >> 2) * (kTile / 2) + (kk & 3) * 32, 16, 1024),
                       tc05::smem_desc_sw128(q_s + (kk >> 2) * (kQ / 2) + (kk & 3) * 32, 16, 1024), idS,
                       kk > 0 ? 1u : 0u);
        tc05::mma_commit(&bars.sfull[j & 1]);
        tc05::mma_commit(&bars.kempty[st]);
      };
      int ns = 0;  // S^T issued for tiles < ns
      bool ok = true;
      for (int i = 0; ok && i < n; ++i) {
        bool p_ready = false, v_ready = false;
        for (uint32_t it = 0;; ++it) {
          const int ns0 = ns;
          if (ns < n && ns <= i + 2 && s_ready(ns)) issue_S(ns++);
          if (ns > i) {
            v_ready = v_ready || mbar_test_wait(&bars.vfull[i % kVStages], (i / kVStages) & 1);
            p_ready = v_ready && mbar_test_wait(&bars.pfull, i & 1);
            if (p_ready) break;
          }
          if (ns == ns0) poll_pause();
          if (it >= kWaitSpinLimit) { *abort = 1; ok = false; break; }
          if ((it & 31u) == 31u && *abort) { ok = false; break; }
        }
        if (!ok) break;
        tc05::fence_after_sync();
        const int st = i % kVStages;
        const uint32_t v_s = smem_u32(sV(st)), p_s = smem_u32(sP);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc05::mma_ss(tmem + 64, tc05::smem_desc_sw128(v_s + kk * 2048, kTile / 2, 1024),
                       tc05::smem_desc_sw128(p_s + kk * 2048, kTile / 2, 1024), idO,
                       (i > 0 || kk > 0) ? 1u : 0u);
        tc05::mma_commit(&bars.pfree);
        tc05::mma_commit(&bars.vempty[st]);
        if (i == n - 1) tc05::mma_commit(&bars.ofull);
      }
      tc05::mma_commit(&bars.done);  // arrives once every MMA issued above has completed
    }
  } else {
    // ---------------------------------------------------------------- softmax, one key per thread
    // Two warpgroups: warp w takes keys 32 (w % 4) .. + 31 of each tile (its TMEM lane quarter)
    // and the 16 queries 16 qh .. + 15 of its group qh, so a tile's exponentials and P stores
    // are spread over 8 warps, two per SM sub-partition.  Every wait in front of a warp-collective
    // instruction is voted across the warp, and all eight warps run the same sequence of named
    // barriers whatever happens, so after a timeout they keep walking their tiles without doing
    // work and no barrier waits on a warp that left.
    const int quarter = warp & 3;
    const int L = 32 * quarter + lane;  // key of the tile (S^T lane) and column d of O (O^T lane)
    const uint32_t lane_off = uint32_t(32 * quarter) << 16;
    const int wr = warp - 2;            // this warp's row of bars.red (0-7)
    const int qh = wr >> 2, q0 = 16 * qh;
    const int st_i = int(threadIdx.x) - 64;  // this thread among the 256 softmax threads
    const float c = a.scale_log2;
    if (k > 1 && wr == 0 && lane < a.n_act) {
      // row q = lane of this CTA's partial goes to slot `rank` of its owner's receive region
      // (read at the merge, after several softmax barriers)
      int r = 0;
      while ((r + 1) * a.n_act / k <= lane) ++r;
      const int r0 = r * a.n_act / k, rows = (r + 1) * a.n_act / k - r0;
      bars.row_owner[lane] = r;
      bars.row_off[lane] = (rank * rows + (lane - r0)) * 512;
      bars.ml_off[lane] = k * rows * 512 + (rank * rows + (lane - r0)) * 8;
    }
    bool ok = true;
    float m[16], l[16];  // query q0 + q: reference max and this thread's share of the row sum
#pragma unroll
    for (int q = 0; q < 16; ++q) m[q] = -INFINITY, l[q] = 0.f;
    for (int i = 0; i < n; ++i) {
      const int t = t0 + i;
      ok = __all_sync(FULL, ok && wait_or_abort(&bars.sfull[i & 1], (i >> 1) & 1, abort));
      uint32_t sr[16];
      if (ok) {
        tc05::fence_after_sync();
        tc05::tmem_ld16(tmem + 32 * (i & 1) + q0 + lane_off, sr);
        tc05::tmem_wait_ld();
      } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) sr[q] = 0u;
      }
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.sfree[i & 1]);
      const bool kv = t != 0 || L < a.n_act;  // keys past n_act in the action tile are padding
      if (i == 0) {
        // Every query's first reference: its score against key 0 (a valid key of every tile),
        // so that the exact tile maxima below are taken only for a score more than 2^16 above it
        // (with -inf they always were, a reduction across the 128 keys on every CTA's first
        // tile).  Any finite reference gives the same result; only its headroom matters.
        if (L == 0) {
#pragma unroll
          for (int q = 0; q < 16; ++q) bars.red[qh][q] = __uint_as_float(sr[q]) * c;
        }
        softmax8_sync();
#pragma unroll
        for (int q = 0; q < 16; ++q) m[q] = bars.red[qh][q];
        softmax8_sync();  // bars.red is rewritten below
      }
      float ymax = -INFINITY;
#pragma unroll
      for (int q = 0; q < 16; ++q) ymax = fmaxf(ymax, fmaf(__uint_as_float(sr[q]), c, -m[q]));
      if (softmax8_any(ok && kv && !(ymax <= kLazy))) {
        // Some query's reference must move: the tile's max per query over its valid keys (the
        // four warps of the group, one lane quarter each).
        float v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] = kv ? __uint_as_float(sr[q]) * c : -INFINITY;
        const float red = reduce_scatter16<true>(v, lane);
        if (lane < 16) bars.red[wr][lane] = red;
        softmax8_sync();
        float al[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float tm = fmaxf(fmaxf(bars.red[4 * qh][q], bars.red[4 * qh + 1][q]),
                                 fmaxf(bars.red[4 * qh + 2][q], bars.red[4 * qh + 3][q]));
          const float mn = tm > m[q] + kLazy ? tm : m[q];
          al[q] = tc05::fast_exp2(m[q] - mn);  // 0 when m was -inf, 1 when it stays
          l[q] *= al[q];
          m[q] = mn;
        }
        if (i > 0) {  // O^T holds the P V of the earlier tiles: rescale its columns of this group
          ok = __all_sync(FULL, ok && wait_or_abort(&bars.pfree, (i - 1) & 1, abort));
          if (ok) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {  // the P_hi and P_lo column blocks
              uint32_t o[16];
              tc05::tmem_ld16(tmem + 64 + 32 * half + q0 + lane_off, o);
              tc05::tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 16; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * al[q]);
              tc05::tmem_st16(tmem + 64 + 32 * half + q0 + lane_off, o);
            }
            tc05::tmem_wait_st();
          }
        }
        softmax8_sync();  // bars.red is rewritten by the next tile
      }
      // P = P_hi + P_lo, both bf16: query columns 0-31 of the P^T row hold P_hi and columns
      // 32-63 P_lo, so the one N = 64 MMA accumulates both and O^T's two column halves add up
      // to P V with P carried to ~16 significant bits (the cache itself is bf16 already).
      uint32_t pk[8], pl[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float p0 = kv ? tc05::fast_exp2(fmaf(__uint_as_float(sr[2 * j]), c, -m[2 * j])) : 0.f;
        const float p1 = kv ? tc05::fast_exp2(fmaf(__uint_as_float(sr[2 * j + 1]), c, -m[2 * j + 1])) : 0.f;
        l[2 * j] += p0, l[2 * j + 1] += p1;
        pk[j] = pack_bf16(p0, p1);  // query q0 + 2j in the low half
        pl[j] = pack_bf16(p0 - __uint_as_float(pk[j] << 16), p1 - __uint_as_float(pk[j] & 0xffff0000u));
      }
      // this group's 32 bytes of P_hi and of P_lo in P^T row L (the 128-byte-swizzled layout the
      // MMA descriptor names: 16-byte chunk ch at (ch ^ (L % 8)) x 16), once P V of the previous
      // tile has read the buffer
      if (i > 0) ok = __all_sync(FULL, ok && wait_or_abort(&bars.pfree, (i - 1) & 1, abort));
      if (ok) {
        uint8_t* row = sP + L * 128;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int ch = 2 * qh + cc;
          *reinterpret_cast<uint4*>(row + ((ch ^ (L & 7)) << 4)) =
              make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
          *reinterpret_cast<uint4*>(row + (((ch + 4) ^ (L & 7)) << 4)) =
              make_uint4(pl[4 * cc], pl[4 * cc + 1], pl[4 * cc + 2], pl[4 * cc + 3]);
        }
      }
      tc05::fence_proxy_async_smem();  // P^T (generic stores) and O^T (tcgen05.st) before the MMA
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.pfull);
    }
    // ---- slice done: the row sums over all 128 keys (while the last P V runs), then O^T
    // column d = L of this thread, for the group's 16 queries
    {
      float v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) v[q] = l[q];
      const float red = reduce_scatter16<false>(v, lane);
      if (lane < 16) bars.red[wr][lane] = red;
    }
    softmax8_sync();
    float lt[16];
#pragma unroll
    for (int q = 0; q < 16; ++q)
      lt[q] = (bars.red[4 * qh][q] + bars.red[4 * qh + 1][q]) + (bars.red[4 * qh + 2][q] + bars.red[4 * qh + 3][q]);
    float o[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) o[q] = 0.f;
    if (n > 0) {
      ok = __all_sync(FULL, ok && wait_or_abort(&bars.ofull, 0, abort));
      if (ok) {
        uint32_t ohi[16], olo[16];
        tc05::fence_after_sync();
        tc05::tmem_ld16(tmem + 64 + q0 + lane_off, ohi);
        tc05::tmem_ld16(tmem + 96 + q0 + lane_off, olo);
        tc05::tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q) o[q] = __uint_as_float(ohi[q]) + __uint_as_float(olo[q]);
      }
    }
    if (k == 1) {
      // the whole (b, h) in this CTA: O = O^T / l
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if (q0 + q >= a.n_act) continue;
        const int64_t off = ((int64_t(b) * a.n_act + q0 + q) * a.H + h) * 128 + L;
        const float val = o[q] / lt[q];
        if (a.o_f32) static_cast<float*>(a.o)[off] = val;
        else static_cast<__nv_bfloat16*>(a.o)[off] = __float2bfloat16_rn(val);
      }
    } else {
      // ---- the merge over the cluster.  Row q of this CTA's partial goes to slot `rank` of the
      // receive region of the row's owner, 16 bytes per st.async counted on the owner's rx_full
      // (armed at the start with every byte it will receive); this CTA's own rows are copied
      // locally.  The P^T buffer (every P V is done) stages the partial as [32 queries][128].
      float* part = reinterpret_cast<float*>(sP);
#pragma unroll
      for (int q = 0; q < 16; ++q) part[(q0 + q) * 128 + L] = o[q];
      if (quarter == 0 && lane < 16) {  // one warp of each group: its queries' (m, l)
        float mm = -INFINITY, ll = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (q == lane) mm = m[q], ll = lt[q];
        bars.part_m[q0 + lane] = mm;
        bars.part_l[q0 + lane] = ll;
      }
      softmax8_sync();
      asm volatile("barrier.cluster.wait.acquire;" ::: "memory");  // every owner has armed rx_full
#pragma unroll 1
      for (int it = 0; it < 4; ++it) {  // chunk c: 16 bytes of row c / 32 (n_act <= 32 rows)
        const int cidx = st_i + 256 * it, q = cidx >> 5, ch = cidx & 31;
        if (q >= a.n_act) continue;
        const int r = bars.row_owner[q];
        const float4 v = *reinterpret_cast<const float4*>(part + q * 128 + 4 * ch);
        uint8_t* dst = rx + bars.row_off[q] + 16 * ch;
        if (r == rank) *reinterpret_cast<float4*>(dst) = v;
        else st_async4(peer_addr(dst, uint32_t(r)), v, peer_addr(&bars.rx_full, uint32_t(r)));
      }
      if (st_i < a.n_act) {
        const int r = bars.row_owner[st_i];
        uint8_t* dst = rx + bars.ml_off[st_i];
        if (r == rank) *reinterpret_cast<float2*>(dst) = make_float2(bars.part_m[st_i], bars.part_l[st_i]);
        else st_async2(peer_addr(dst, uint32_t(r)), bars.part_m[st_i], bars.part_l[st_i], peer_addr(&bars.rx_full, uint32_t(r)));
      }
      wait_cluster(&bars.rx_full, 0, abort);  // every peer's rows for this CTA have landed
      softmax8_sync();                        // and this CTA's own copies
      // merge rows [r0, r1): warp wr takes rows wr, wr + 8, ... (one round for rows <= 8), lane l
      // the columns 4 l .. 4 l + 3; lane p < k loads slot p's (m, l) pair and the warp shares
      // its weight, so each thread loads one 16-byte chunk per slot and takes one exponential
      const int r0 = rank * a.n_act / k, r1 = (rank + 1) * a.n_act / k, rows = r1 - r0;
      const float* rxo = reinterpret_cast<const float*>(rx);
      const float* rml = reinterpret_cast<const float*>(rx + k * rows * 512);
      // (the merge and the sends above run once per CTA, from a cold instruction cache: their
      // loops stay rolled)
      for (int j = wr; j < rows; j += 8) {
        const float2 ml = lane < k ? *reinterpret_cast<const float2*>(rml + 2 * (lane * rows + j))
                                   : make_float2(-INFINITY, 0.f);
        float M = ml.x;  // max over lanes 0 .. 7 (k <= 8), then lane 0's to all
        M = fmaxf(M, __shfl_xor_sync(FULL, M, 1));
        M = fmaxf(M, __shfl_xor_sync(FULL, M, 2));
        M = fmaxf(M, __shfl_xor_sync(FULL, M, 4));
        M = __shfl_sync(FULL, M, 0);
        const float Mu = M == -INFINITY ? 0.f : M;
        const float wl = lane < k ? tc05::fast_exp2(ml.x - Mu) : 0.f;  // slot `lane`'s weight
        float den = wl * ml.y;
        den += __shfl_xor_sync(FULL, den, 1);
        den += __shfl_xor_sync(FULL, den, 2);
        den += __shfl_xor_sync(FULL, den, 4);
        den = __shfl_sync(FULL, den, 0);
        float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
        for (int p = 0; p < k; ++p) {
          const float wgt = __shfl_sync(FULL, wl, p);
          const float4 x = *reinterpret_cast<const float4*>(rxo + (p * rows + j) * 128 + 4 * lane);
          num.x = fmaf(wgt, x.x, num.x), num.y = fmaf(wgt, x.y, num.y);
          num.z = fmaf(wgt, x.z, num.z), num.w = fmaf(wgt, x.w, num.w);
        }
        const float inv = den > 0.f ? __fdividef(1.f, den) : 0.f;
        const int64_t off = ((int64_t(b) * a.n_act + r0 + j) * a.H + h) * 128 + 4 * lane;
        if (a.o_f32)
          *reinterpret_cast<float4*>(static_cast<float*>(a.o) + off) =
              make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
        else
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.o) + off) =
              make_uint2(pack_bf16(num.x * inv, num.y * inv), pack_bf16(num.z * inv, num.w * inv));
      }
    }
  }
  // the producer and MMA warps close their phase of the cluster barrier before leaving
  if (k > 1 && warp < 2) asm volatile("barrier.cluster.wait;" ::: "memory");

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  tc05::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    mbar_wait(&bars.done, 0);  // every MMA has completed (bounded)
    tc05::fence_after_sync();
    tc05::tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && bars.abort && a.err) atomicExch(a.err, int(WAM_ERR_TIMEOUT));
}

// The part of the call a CTA of the 128-key reads owns: episode b, head h, part r of k, i.e. the
// video tiles [1 + r nv / k, 1 + (r + 1) nv / k) of (b, h), and the action tile for r = 0.  Consecutive CTAs take the same part of consecutive
// heads, so the CTAs reading at one moment cover the same token range of every head (one fused
// K or V token row holds all heads, H x 256 bytes).
__device__ __forceinline__ void aligned_part(const ActionArgs& a, int cta, int& b, int& h, int& r, int& k) {
  b = 0;
  for (;;) {
    k = a.kparts[b];
    const int n_c = a.H * k;
    if (cta < n_c || b == a.B - 1) break;
    cta -= n_c;
    ++b;
  }
  r = cta / a.H;
  h = cta % a.H;
}

// End of one segment of a split read, in the 128 softmax threads (thread L = column d of O):
// o[q] is the segment's unnormalised O^T column, lt[q] its row sums and m[q] its reference maxima
// (log2 units, the same in every thread).  A segment that covers its whole (episode, head)
// (parts == 1) writes O = o / lt.  Otherwise it stores a partial (O [32 queries][128], m [32],
// l [32]) in its workspace slot and takes a ticket; the last of the (episode, head)'s parts to
// arrive merges every partial, its own included, in slot order (so the result does not depend
// on the arrival order), writes O and resets the ticket.  The merge brings all partials into
// shared memory at once with bulk copies (`stage`, room for `stage_parts` of them: the K/V ring,
// idle by then; `mbar` an mbarrier of the CTA used only here) and merges from there: warp 0 turns
// the maxima into per-part weights, then each warp combines 8 query rows, 4 columns per lane.
// More parts than the stage holds are merged from global memory one part at a time.  `last` is a
// shared word of the CTA.
__device__ __forceinline__ void split_finish_segment(const ActionArgs& a, int b, int h, int parts,
                                                     int slot, int L, int wr, int lane,
                                                     float (&o)[32], float (&lt)[32],
                                                     float (&m)[32], int* last, uint8_t* stage,
                                                     int stage_parts, uint64_t* mbar,
                                                     volatile int* abort) {
  const int bh = b * a.H + h;
  if (parts == 1) {
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      if (q >= a.n_act) continue;
      const int64_t off = ((int64_t(b) * a.n_act + q) * a.H + h) * 128 + L;
      const float val = o[q] / lt[q];
      if (a.o_f32) static_cast<float*>(a.o)[off] = val;
      else static_cast<__nv_bfloat16*>(a.o)[off] = __float2bfloat16_rn(val);
    }
    return;
  }
  const float* part0 = a.ws_part + int64_t(bh) * a.max_parts * kSlotFloats;
  float* mine = a.ws_part + (int64_t(bh) * a.max_parts + slot) * kSlotFloats;
#pragma unroll
  for (int q = 0; q < 32; ++q) __stcg(mine + q * 128 + L, o[q]);  // row q: one warp, 128 bytes
  if (wr == 0) {
    float mm = -INFINITY, ll = 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q)
      if (q == lane) mm = m[q], ll = lt[q];
    __stcg(mine + 4096 + lane, mm);
    __stcg(mine + 4096 + 32 + lane, ll);
  }
  // the CTA's stores, ordered before one thread's release of the ticket by the CTA barrier (the
  // fence is cumulative), so only that thread fences
  um::softmax_sync();
  if (wr == 0 && lane == 0) {
    __threadfence();
    const int prev = atomicAdd(a.ws_count + bh, 1);
    __threadfence();
    *reinterpret_cast<volatile int*>(last) = prev == parts - 1;
  }
  um::softmax_sync();
  if (!*reinterpret_cast<volatile int*>(last)) return;

  if (parts <= stage_parts) {
    // every partial into shared memory (the other parts' writes were made visible before their
    // tickets; this CTA's acquire above orders them before the async-proxy reads)
    constexpr uint32_t kSlotBytes = uint32_t(kSlotFloats) * 4u;
    if (wr == 0 && lane == 0) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      mbar_arrive_expect_tx(mbar, kSlotBytes * uint32_t(parts));
      for (int p = 0; p < parts; ++p)
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                smem_u32(stage + p * kSlotBytes)),
            "l"(part0 + int64_t(p) * kSlotFloats), "r"(kSlotBytes), "r"(smem_u32(mbar))
            : "memory");
    }
    if (!mbar_wait(mbar, 0)) {  // bounded: a wait that gives up reports a timeout, O is not written
      *abort = 1;
      return;
    }
    const float* sp = reinterpret_cast<const float*>(stage);
    float* wts = reinterpret_cast<float*>(stage + parts * kSlotBytes);  // [parts][32], then 1 / l [32]
    if (wr == 0) {
      const int q = lane;
      float M = -INFINITY;
      for (int p = 0; p < parts; ++p) M = fmaxf(M, sp[p * kSlotFloats + 4096 + q]);
      float den = 0.f;
      for (int p = 0; p < parts; ++p) {
        const float w = tc05::fast_exp2(sp[p * kSlotFloats + 4096 + q] - M);
        wts[p * 32 + q] = w;
        den = fmaf(w, sp[p * kSlotFloats + 4096 + 32 + q], den);
      }
      wts[parts * 32 + q] = den > 0.f ? 1.f / den : 0.f;
    }
    um::softmax_sync();
    for (int q = wr; q < a.n_act; q += 4) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int p = 0; p < parts; ++p) {
        const float w = wts[p * 32 + q];
        const float4 x = *reinterpret_cast<const float4*>(sp + p * kSlotFloats + q * 128 + 4 * lane);
        acc.x = fmaf(w, x.x, acc.x), acc.y = fmaf(w, x.y, acc.y);
        acc.z = fmaf(w, x.z, acc.z), acc.w = fmaf(w, x.w, acc.w);
      }
      const float inv = wts[parts * 32 + q];
      const int64_t off = ((int64_t(b) * a.n_act + q) * a.H + h) * 128 + 4 * lane;
      if (a.o_f32) {
        *reinterpret_cast<float4*>(static_cast<float*>(a.o) + off) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      } else {
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.o) + off) =
            make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
      }
    }
  } else {
    // more parts than the stage holds: thread L merges its column part by part from global memory
#pragma unroll
    for (int q = 0; q < 32; ++q) o[q] = 0.f, lt[q] = 0.f, m[q] = -INFINITY;
    for (int p = 0; p < parts; ++p) {
      const float* ps = part0 + int64_t(p) * kSlotFloats;
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const float pm = __ldcg(ps + 4096 + q), pz = __ldcg(ps + 4096 + 32 + q), po = __ldcg(ps + q * 128 + L);
        const float mn = fmaxf(m[q], pm);
        const float fa = tc05::fast_exp2(m[q] - mn), fb = tc05::fast_exp2(pm - mn);
        o[q] = fmaf(o[q], fa, po * fb);
        lt[q] = fmaf(lt[q], fa, pz * fb);
        m[q] = mn;
      }
    }
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      if (q >= a.n_act) continue;
      const int64_t off = ((int64_t(b) * a.n_act + q) * a.H + h) * 128 + L;
      const float val = lt[q] > 0.f ? o[q] / lt[q] : 0.f;
      if (a.o_f32) static_cast<float*>(a.o)[off] = val;
      else static_cast<__nv_bfloat16*>(a.o)[off] = __float2bfloat16_rn(val);
    }
  }
  if (wr == 0 && lane == 0) a.ws_count[bh] = 0;  // ready for the next call
}

// ============================================================================================
// The fused read over an NVFP4 cache (wam_action_attn_nvfp4): codes, E4M3 block scales and a
// tensor scale per fused K or V, head-major, as wam_fused_to_nvfp4 writes them.  Same work split,
// merge and online softmax as the split read; what changes is how a K or V tile reaches shared
// memory and the operand type:
//  - the producer copies a video tile's 8 KB of codes and 1 KB of scales with two bulk copies into
//    a raw ring (3 slots for K, 3 for V); one converter warp for K (warp 6) and one for V
//    (warp 7) decode e2m1 x e4m3 into fp16, exactly (a product has at most 6 significant bits),
//    in the 128-byte-swizzled layout the MMA descriptors name;
//  - the action tile and the Q tile arrive in bf16 by TMA and are converted in place to fp16;
//  - both MMAs run on fp16 operands (P = P_hi + P_lo in fp16; the reference headroom is 2^15 so
//    P stays below fp16's largest finite value);
//  - the tensor scales stay outside the MMAs: a video tile's scores are multiplied by s_g(K) in
//    the softmax, and the video tiles' P V accumulate apart from the action tile's (two O^T
//    buffers per segment), combined at the end as s_g(V) O_video + O_action.
namespace fq {
constexpr int kKeys = 128;
constexpr int kTile = kKeys * 128 * 2;   // one fp16 K or V tile: 32 KB
constexpr int kStages = 2;               // fp16 K and V tiles
constexpr int kRaw = 2;                  // raw slots for K and for V
constexpr int kCodes = kKeys * 64;       // codes of one tile: 8 KB
constexpr int kScales = kKeys * 8;       // E4M3 scales of one tile: 1 KB
constexpr int kRawBytes = kCodes + kScales;
constexpr int kQ = 32 * 128 * 2;
constexpr int kP = kKeys * 128;
// Warpgroups: 0 = producer (warp 0), MMA issuer (warp 1), two idle warps; 1 = softmax; 2 = K (and
// Q) converters; 3 = V converters.  The softmax warpgroup holds 32 running maxima and sums per
// thread, so the registers are split unevenly (setmaxnreg); the shares add up to the block's
// launch allocation of 128 per thread.
constexpr int kThreads = 16 * 32;
constexpr int kConvWarps = 4;
constexpr uint32_t kRegsCtl = 80, kRegsSoftmax = 256, kRegsConv = 88, kRegsLaunch = 128;
static_assert(kRegsCtl + kRegsSoftmax + 2 * kRegsConv == 4 * kRegsLaunch, "register split");
constexpr uint32_t kTmemCols = 512;      // S^T 0, 32; O^T video 64 + 64 p; O^T action 192 + 64 p
constexpr float kLazy = 15.f;            // P <= 2^15 < 65504
struct Bars {
  uint64_t qland[2], qfull[2], qempty[2];
  uint64_t kland[kStages], kfull[kStages], kempty[kStages];
  uint64_t vland[kStages], vfull[kStages], vempty[kStages];
  uint64_t rkfull[kRaw], rkfree[kRaw], rvfull[kRaw], rvfree[kRaw];
  uint64_t sfull[2], sfree[2], pfull[2], pfree[2], ofull[2], ofree[2], done;
  uint64_t mfull;
  uint32_t tmem_base;
  int abort;
  int last;
  int part_r, part_k;
  float red[4][32];
};
constexpr int kSmemBytes =
    1024 + 2 * kQ + kStages * 2 * kTile + 2 * kRaw * kRawBytes + 2 * kP + int(sizeof(Bars)) + 64;
static_assert(kSmemBytes <= 232448, "shared memory");
// partials the fp16 K/V stages and the raw rings (contiguous) hold for the merge
constexpr int kStageParts = (kStages * 2 * kTile + 2 * kRaw * kRawBytes - 128) / (kSlotFloats * 4 + 128);

// Instruction descriptor of .kind::f16 with fp16 A and B and an fp32 accumulator (format 0).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool b_mn_major, bool a_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
// Bulk copy global -> shared (contiguous, 16-byte aligned, multiple of 16 bytes), counted on an
// mbarrier; no multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// 16 bytes of bf16 (8 elements) -> 16 bytes of fp16, in place.
__device__ __forceinline__ void bf16_to_f16_chunk(uint8_t* p) {
  uint4 u = *reinterpret_cast<uint4*>(p);
  uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = pack_f16(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
// A whole bf16 tile of `bytes` converted in place by `nt` threads (thread t of them).
__device__ __forceinline__ void bf16_tile_to_f16(uint8_t* tile, int bytes, int t, int nt) {
  for (int c = t; c < bytes / 16; c += nt) bf16_to_f16_chunk(tile + 16 * c);
}
// Eight E2M1 codes of one word (element 2i in the low nibble of byte i) -> four fp16 pairs
// (pair i = elements 2i, 2i + 1, the first in the low half): one unpack, four conversions.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t word, uint32_t (&out)[4]) {
  asm("{ .reg .b8 b0, b1, b2, b3;\n"
      " mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(word));
}
// An E4M3 code -> its value as an fp16 pair (both halves).
__device__ __forceinline__ uint32_t e4m3_to_f16x2(uint32_t code) {
  uint32_t r;
  asm("{ .reg .b16 c; cvt.u16.u32 c, %1; cvt.rn.f16x2.e4m3x2 %0, c; }" : "=r"(r) : "r"(code | (code << 8)));
  return r;
}
__device__ __forceinline__ uint32_t mul_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// 16 bytes of codes (32 elements: blocks 2 q and 2 q + 1 of key row r) of a raw tile and the 4
// scale bytes of those blocks.  A warp instruction covers 8 rows x 4 chunks; 16-byte accesses
// are served by quarter-warps of 8 lanes, so the lanes of each quarter take rows and chunks that
// fall in 8 different 16-byte bank groups both for the loads (row r, chunk q of 64-byte code
// rows: group 4 (r & 1) + q) and for the stores into the swizzled fp16 tile (chunks 0 and 4 of
// a 64-column half XOR r & 7): quarter p takes rows 4 (p / 2) .. +3, pairs of rows with chunks
// {0, 1} and {2, 3}, swapped for odd p.
__device__ __forceinline__ int chunk_row(int lane) {
  const int p = lane >> 3, k = lane & 7;
  return 4 * (p >> 1) + 2 * (k >> 2) + (k & 1);
}
__device__ __forceinline__ int chunk_q(int lane) {
  const int p = lane >> 3, k = lane & 7;
  return (((k >> 1) & 1) | ((k >> 2) << 1)) ^ ((p & 1) << 1);
}
struct RawChunk {
  uint4 c;
  uint32_t sw;
};
__device__ __forceinline__ RawChunk load_chunk(const uint8_t* raw, int r, int q) {
  RawChunk x;
  x.c = *reinterpret_cast<const uint4*>(raw + r * 64 + q * 16);
  x.sw = *reinterpret_cast<const uint32_t*>(raw + kCodes + r * 8 + (q >> 1) * 4);
  return x;
}
// The chunk decoded (code value times its block's scale, in fp16) into the swizzled fp16 tile.
__device__ __forceinline__ void store_chunk(const RawChunk& x, uint8_t* tile, int r, int q) {
  const uint32_t cw[4] = {x.c.x, x.c.y, x.c.z, x.c.w};
#pragma unroll
  for (int half = 0; half < 2; ++half) {  // one 16-element block, two 8-element chunks
    const int blk = 2 * q + half;
    const uint32_t s2 = e4m3_to_f16x2((x.sw >> (8 * (blk & 3))) & 0xFFu);
    uint32_t out[8];
    e2m1x8_to_f16x2(cw[2 * half], *reinterpret_cast<uint32_t(*)[4]>(&out[0]));
    e2m1x8_to_f16x2(cw[2 * half + 1], *reinterpret_cast<uint32_t(*)[4]>(&out[4]));
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = mul_f16x2(out[e], s2);
    const int ch0 = 2 * blk;  // 8-element chunks 2 blk and 2 blk + 1 of the row
    *reinterpret_cast<uint4*>(tile + swz128<128>(r, 8 * ch0)) = make_uint4(out[0], out[1], out[2], out[3]);
    *reinterpret_cast<uint4*>(tile + swz128<128>(r, 8 * ch0 + 8)) = make_uint4(out[4], out[5], out[6], out[7]);
  }
}
// The row groups g, g + 4, g + 8, g + 12 (of 16 groups of 8 rows) of a raw tile decoded by warp g of
// the four converter warps: all loads first, so that the warp has four chunks in flight.
__device__ __forceinline__ void decode_rows(const uint8_t* raw, uint8_t* tile, int g, int lane) {
  const int rr = chunk_row(lane), q = chunk_q(lane);
  RawChunk x[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] = load_chunk(raw, 8 * (g + 4 * j) + rr, q);
#pragma unroll
  for (int j = 0; j < 4; ++j) store_chunk(x[j], tile, 8 * (g + 4 * j) + rr, q);
}
template <uint32_t R>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
}  // namespace fq

__global__ void __launch_bounds__(fq::kThreads, 1)
action_nvfp4_kernel(const __grid_constant__ ActionArgs a, const __grid_constant__ ActionMaps maps) {
  using namespace fq;
  if (threadIdx.x == 0) prefetch_tmap(&maps.q), prefetch_tmap(&maps.ka), prefetch_tmap(&maps.va);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  auto sQ = [&](int s) { return base + (s & 1) * kQ; };
  auto sK = [&](int st) { return base + 2 * kQ + st * 2 * kTile; };
  auto sV = [&](int st) { return base + 2 * kQ + st * 2 * kTile + kTile; };
  auto rK = [&](int sl) { return base + 2 * kQ + kStages * 2 * kTile + sl * kRawBytes; };
  auto rV = [&](int sl) { return base + 2 * kQ + kStages * 2 * kTile + (kRaw + sl) * kRawBytes; };
  // P^T of tile i in buffer i % 2, so that the softmax writes tile i while the MMA reads tile i - 1
  uint8_t* sP0 = base + 2 * kQ + kStages * 2 * kTile + 2 * kRaw * kRawBytes;
  auto sP = [&](int i) { return sP0 + (i & 1) * kP; };
  fq::Bars& bars = *reinterpret_cast<fq::Bars*>(sP0 + 2 * kP);
  volatile int* abort = &bars.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned FULL = 0xffffffffu;
  int part_b, part_h, part_r, part_k;
  aligned_part(a, int(blockIdx.x), part_b, part_h, part_r, part_k);
  // the video tiles 1 .. nv of (b, h) cut evenly; part 0 also takes the action tile (t = 0)
  const int part_nv = tiles_of<kKeys>(a, part_b) - 1;
  const int t0 = part_r == 0 ? 0 : 1 + part_r * part_nv / part_k;
  const int n = 1 + (part_r + 1) * part_nv / part_k - t0;  // n >= 1: k <= nv
  const int tpf = a.T / kKeys;
  const int64_t N = int64_t(a.F) * a.T;
  // head-major row of the first key of video tile t of (b, h)
  auto raw_row = [&](const TileWalk<kKeys>& w) {
    const int vt = w.t - 1;
    const int64_t tok = int64_t(a.fl.vlist[w.b * a.F + vt / tpf]) * a.T + (vt % tpf) * kKeys;
    return (int64_t(w.b) * a.H + w.h) * N + tok;
  };
  uint32_t pre = 0;  // bit i: raw tile i of the part requested before the dependency wait

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.qland[i], 1);
      mbar_init(&bars.qfull[i], kConvWarps);
      mbar_init(&bars.qempty[i], 1);
      mbar_init(&bars.sfull[i], 1);
      mbar_init(&bars.sfree[i], 4);
      mbar_init(&bars.ofull[i], 1);
      mbar_init(&bars.ofree[i], 4);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars.kland[i], 1);
      mbar_init(&bars.kfull[i], kConvWarps);
      mbar_init(&bars.kempty[i], 1);
      mbar_init(&bars.vland[i], 1);
      mbar_init(&bars.vfull[i], kConvWarps);
      mbar_init(&bars.vempty[i], 1);
    }
    for (int i = 0; i < kRaw; ++i) {
      mbar_init(&bars.rkfull[i], 1);
      mbar_init(&bars.rkfree[i], kConvWarps);
      mbar_init(&bars.rvfull[i], 1);
      mbar_init(&bars.rvfree[i], kConvWarps);
    }
    mbar_init(&bars.pfull[0], 4);
    mbar_init(&bars.pfull[1], 4);
    mbar_init(&bars.pfree[0], 1);
    mbar_init(&bars.pfree[1], 1);
    mbar_init(&bars.done, 1);
    bars.abort = 0;
    bars.last = 0;
    bars.part_r = part_r, bars.part_k = part_k;
    mbar_init(&bars.mfull, 1);
    fence_barrier_init();
    // Up to here only this CTA's shared memory was touched.  With a.fused_ready (the previous
    // kernel does not write the NVFP4 pair) the part's first raw tiles are requested now, by
    // the thread that set up their barriers, before the block-wide sync and the dependency wait.
    if (a.fused_ready) {
      TileWalk<kKeys> w;
      w.init_at(a, part_b, part_h, t0);
      for (int i = 0, r = 0; i < n && r < kRaw; ++i, w.next(a)) {
        if (w.t == 0) continue;
        const int64_t row = raw_row(w);
        mbar_arrive_expect_tx(&bars.rkfull[r], kRawBytes);
        bulk_load(rK(r), a.k_codes + row * 64, kCodes, &bars.rkfull[r]);
        bulk_load(rK(r) + kCodes, a.k_scales + row * 8, kScales, &bars.rkfull[r]);
        mbar_arrive_expect_tx(&bars.rvfull[r], kRawBytes);
        bulk_load(rV(r), a.v_codes + row * 64, kCodes, &bars.rvfull[r]);
        bulk_load(rV(r) + kCodes, a.v_scales + row * 8, kScales, &bars.rvfull[r]);
        pre |= 1u << i;
        ++r;
      }
    }
  }
  if (warp == 1) {
    tc05::tmem_alloc(&bars.tmem_base, kTmemCols);
    tc05::tmem_relinquish();
  }
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = bars.tmem_base;
  grid_dependency_wait();
  grid_launch_dependents();
  // One register share per warpgroup, taken by all four of its warps at the top of its branch.
  if (warp < 4) {
    regs_dec<kRegsCtl>();
    if (warp == 0) {
      // ---------------------------------------------------------------- producer
      if (lane == 0) {
        TileWalk<kKeys> kw, vw;
        kw.init_at(a, part_b, part_h, t0);
        vw.init_at(a, part_b, part_h, t0);
        int nk = 0, nv = 0, kseg = -1, rk = 0, rv = 0;
        int kact[kStages] = {0, 0}, vact[kStages] = {0, 0};
        for (uint32_t it = 0; (nk < n || nv < n) && it < kWaitSpinLimit; ++it) {
          if ((it & 31u) == 31u && *abort) break;
          const int nk0 = nk, nv0 = nv;
          if (nk < n) {
            const bool new_seg = nk == 0 || kw.t == 0, act = kw.t == 0;
            const int s = kseg + 1;
            bool can = !new_seg || s < 2 || mbar_test_wait(&bars.qempty[s & 1], ((s >> 1) - 1) & 1);
            if (act) can = can && (nk < kStages || mbar_test_wait(&bars.kempty[nk % kStages], ((nk / kStages) - 1) & 1));
            else can = can && (rk < kRaw || mbar_test_wait(&bars.rkfree[rk % kRaw], ((rk / kRaw) - 1) & 1));
            if (can) {
              if (new_seg) {
                kseg = s;
                mbar_arrive_expect_tx(&bars.qland[s & 1], kQ);
                tma_load_4d(sQ(s), &maps.q, &bars.qland[s & 1], 0, kw.h, 0, kw.b);
                tma_load_4d(sQ(s) + kQ / 2, &maps.q, &bars.qland[s & 1], 64, kw.h, 0, kw.b);
              }
              if (act) {
                const int st = nk % kStages;
                mbar_arrive_expect_tx(&bars.kland[st], kTile);
                tma_load_4d(sK(st), &maps.ka, &bars.kland[st], 0, kw.h, 0, kw.b);
                tma_load_4d(sK(st) + kTile / 2, &maps.ka, &bars.kland[st], 64, kw.h, 0, kw.b);
                ++kact[st];
              } else {
                const int sl = rk % kRaw;
                if (!(nk < 32 && ((pre >> nk) & 1u))) {  // not requested before the wait
                  const int64_t row = raw_row(kw);
                  mbar_arrive_expect_tx(&bars.rkfull[sl], kRawBytes);
                  bulk_load(rK(sl), a.k_codes + row * 64, kCodes, &bars.rkfull[sl]);
                  bulk_load(rK(sl) + kCodes, a.k_scales + row * 8, kScales, &bars.rkfull[sl]);
                }
                ++rk;
              }
              ++nk;
              kw.next(a);
            }
          }
          if (nv < n) {
            const bool act = vw.t == 0;
            const bool can = act ? (nv < kStages || mbar_test_wait(&bars.vempty[nv % kStages], ((nv / kStages) - 1) & 1))
                                 : (rv < kRaw || mbar_test_wait(&bars.rvfree[rv % kRaw], ((rv / kRaw) - 1) & 1));
            if (can) {
              if (act) {
                const int st = nv % kStages;
                mbar_arrive_expect_tx(&bars.vland[st], kTile);
                tma_load_4d(sV(st), &maps.va, &bars.vland[st], 0, vw.h, 0, vw.b);
                tma_load_4d(sV(st) + kTile / 2, &maps.va, &bars.vland[st], 64, vw.h, 0, vw.b);
                ++vact[st];
              } else {
                const int sl = rv % kRaw;
                if (!(nv < 32 && ((pre >> nv) & 1u))) {
                  const int64_t row = raw_row(vw);
                  mbar_arrive_expect_tx(&bars.rvfull[sl], kRawBytes);
                  bulk_load(rV(sl), a.v_codes + row * 64, kCodes, &bars.rvfull[sl]);
                  bulk_load(rV(sl) + kCodes, a.v_scales + row * 8, kScales, &bars.rvfull[sl]);
                }
                ++rv;
              }
              ++nv;
              vw.next(a);
            }
          }
          if (nk == nk0 && nv == nv0) poll_pause();
        }
        if (nk < n || nv < n) *abort = 1;
        // Copies still in flight land before the CTA leaves (only after an abort can any be).
        for (int i = (rk > kRaw ? rk - kRaw : 0); i < rk; ++i) mbar_wait(&bars.rkfull[i % kRaw], (i / kRaw) & 1);
        for (int i = (rv > kRaw ? rv - kRaw : 0); i < rv; ++i) mbar_wait(&bars.rvfull[i % kRaw], (i / kRaw) & 1);
        for (int st = 0; st < kStages; ++st) {
          if (kact[st]) mbar_wait(&bars.kland[st], (kact[st] - 1) & 1);
          if (vact[st]) mbar_wait(&bars.vland[st], (vact[st] - 1) & 1);
        }
        for (int s = (kseg > 1 ? kseg - 1 : 0); s <= kseg; ++s) mbar_wait(&bars.qland[s & 1], (s >> 1) & 1);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        const uint32_t idS = idesc_f16_f32(128, 32, false, false);
        // N = 32: P is one fp16 part, in query columns 0-31 of each P^T row
        const uint32_t idO = idesc_f16_f32(128, 32, true, true);
        TileWalk<kKeys> sw, pw;
        sw.init_at(a, part_b, part_h, t0);
        pw.init_at(a, part_b, part_h, t0);
        int ns = 0, sseg = -1, pseg = -1;
        bool ok = true, vid_started = false;
        for (int i = 0; ok && i < n; ++i) {
          const bool p_first = i == 0 || pw.t == 0;
          const bool p_last = i == n - 1 || pw.t == pw.nb - 1;
          if (p_first) ++pseg, vid_started = false;
          bool v_ready = false, p_ready = false, o_ready = !(p_first && pseg >= 2);
          for (uint32_t it = 0;; ++it) {
            const int ns0 = ns;
            if (ns < n && ns <= i + 2) {
              const bool s_first = ns == 0 || sw.t == 0;
              const int s = sseg + (s_first ? 1 : 0);
              if (mbar_test_wait(&bars.kfull[ns % kStages], (ns / kStages) & 1) &&
                  (!s_first || mbar_test_wait(&bars.qfull[s & 1], (s >> 1) & 1)) &&
                  (ns < 2 || mbar_test_wait(&bars.sfree[ns & 1], ((ns >> 1) - 1) & 1))) {
                const bool s_last = ns == n - 1 || sw.t == sw.nb - 1;
                sseg = s;
                const int st = ns % kStages;
                tc05::fence_after_sync();
                const uint32_t k_s = smem_u32(sK(st)), q_s = smem_u32(sQ(s));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  tc05::mma_ss(tmem + 32 * (ns & 1),
                               tc05::smem_desc_sw128(k_s + (kk >> 2) * (kTile / 2) + (kk & 3) * 32, 16, 1024),
                               tc05::smem_desc_sw128(q_s + (kk >> 2) * (kQ / 2) + (kk & 3) * 32, 16, 1024), idS,
                               kk > 0 ? 1u : 0u);
                tc05::mma_commit(&bars.sfull[ns & 1]);
                tc05::mma_commit(&bars.kempty[st]);
                if (s_last) tc05::mma_commit(&bars.qempty[s & 1]);
                ++ns;
                sw.next(a);
              }
            }
            if (ns > i) {
              v_ready = v_ready || mbar_test_wait(&bars.vfull[i % kStages], (i / kStages) & 1);
              o_ready = o_ready || mbar_test_wait(&bars.ofree[pseg & 1], ((pseg >> 1) - 1) & 1);
              p_ready = v_ready && o_ready && mbar_test_wait(&bars.pfull[i & 1], (i >> 1) & 1);
              if (p_ready) break;
            }
            if (ns == ns0) poll_pause();
            if (it >= kWaitSpinLimit) { *abort = 1; ok = false; break; }
            if ((it & 31u) == 31u && *abort) { ok = false; break; }
          }
          if (!ok) break;
          tc05::fence_after_sync();
          const int st = i % kStages;
          const bool act = pw.t == 0;
          const uint32_t v_s = smem_u32(sV(st)), p_s = smem_u32(sP(i));
          const uint32_t o_t = tmem + (act ? 192 : 64) + 64 * (pseg & 1);
          const bool acc = !act && vid_started;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc05::mma_ss(o_t, tc05::smem_desc_sw128(v_s + kk * 2048, kTile / 2, 1024),
                         tc05::smem_desc_sw128(p_s + kk * 2048, kTile / 2, 1024), idO,
                         (acc || kk > 0) ? 1u : 0u);
          if (!act) vid_started = true;
          tc05::mma_commit(&bars.pfree[i & 1]);
          tc05::mma_commit(&bars.vempty[st]);
          if (p_last) tc05::mma_commit(&bars.ofull[pseg & 1]);
          pw.next(a);
        }
        tc05::mma_commit(&bars.done);
      }
    }
  } else if (warp < 8) {
    regs_inc<kRegsSoftmax>();
    // ---------------------------------------------------------------- softmax, one key per thread
    const int quarter = warp & 3;
    const int L = 32 * quarter + lane;
    const uint32_t lane_off = uint32_t(32 * quarter) << 16;
    const int wr = warp - 4;
    const float c_act = a.scale_log2, c_vid = a.scale_log2 * *a.k_sg, sg_v = *a.v_sg;
    bool ok = true;
    float m[32], l[32];
    TileWalk<kKeys> tw;
    tw.init_at(a, part_b, part_h, t0);
    int seg = -1, i_first = 0;
    bool has_act = false, has_vid = false;  // accumulators written in this segment so far
    // A P^T row holds P (fp16, kept whole: no low part) in query columns 0-31, the first four
    // 16-byte chunks of its 128-byte swizzled row; the P V MMA reads only those (N = 32).
    for (int i = 0; i < n; ++i, tw.next(a)) {
      if (i == 0 || tw.t == 0) {
        ++seg;
        i_first = i;
        has_act = has_vid = false;
#pragma unroll
        for (int q = 0; q < 32; ++q) m[q] = -INFINITY, l[q] = 0.f;
      }
      const bool last = i == n - 1 || tw.t == tw.nb - 1;
      const bool act = tw.t == 0;
      const float c = act ? c_act : c_vid;
      ok = __all_sync(FULL, ok && um::wait_or_abort(&bars.sfull[i & 1], (i >> 1) & 1, abort));
      uint32_t sr[32];
      if (ok) {
        tc05::fence_after_sync();
        tc05::tmem_ld32(tmem + 32 * (i & 1) + lane_off, sr);
        tc05::tmem_wait_ld();
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) sr[q] = 0u;
      }
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.sfree[i & 1]);
      const bool kv = !act || L < a.n_act;
      const uint32_t o_vid = tmem + 64 + 64 * (seg & 1), o_act = tmem + 192 + 64 * (seg & 1);
      if (i == i_first) {
        // the segment's first reference: each query's score against key 0 (valid in every tile),
        // as in the bf16 read
        if (L == 0) {
#pragma unroll
          for (int q = 0; q < 32; ++q) bars.red[0][q] = __uint_as_float(sr[q]) * c;
        }
        um::softmax_sync();
#pragma unroll
        for (int q = 0; q < 32; ++q) m[q] = bars.red[0][q];
        um::softmax_sync();
      }
      float ymax = -INFINITY;
#pragma unroll
      for (int q = 0; q < 32; ++q) ymax = fmaxf(ymax, fmaf(__uint_as_float(sr[q]), c, -m[q]));
      if (um::softmax_any(ok && kv && !(ymax <= kLazy))) {
        float v[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = kv ? __uint_as_float(sr[q]) * c : -INFINITY;
        bars.red[wr][lane] = um::reduce_scatter32<true>(v, lane);
        um::softmax_sync();
        float al[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float tm = fmaxf(fmaxf(bars.red[0][q], bars.red[1][q]), fmaxf(bars.red[2][q], bars.red[3][q]));
          const float mn = tm > m[q] + kLazy ? tm : m[q];
          al[q] = tc05::fast_exp2(m[q] - mn);
          l[q] *= al[q];
          m[q] = mn;
        }
        if (i > i_first) {  // rescale the accumulators the segment's earlier tiles wrote
          ok = __all_sync(FULL, ok && um::wait_or_abort(&bars.pfree[(i - 1) & 1], ((i - 1) >> 1) & 1, abort));
          if (ok) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {
              if (which == 0 ? !has_vid : !has_act) continue;
              const uint32_t ob = which == 0 ? o_vid : o_act;
              uint32_t o[32];
              tc05::tmem_ld32(ob + lane_off, o);
              tc05::tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * al[q]);
              tc05::tmem_st32(ob + lane_off, o);
            }
            tc05::tmem_wait_st();
          }
        }
        um::softmax_sync();
      }
      // P in fp16 (query columns 0-31 of the P^T row); its rounding (a relative 2^-12) is far
      // inside the read's bf16 tolerance
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float p0 = kv ? tc05::fast_exp2(fmaf(__uint_as_float(sr[2 * j]), c, -m[2 * j])) : 0.f;
        const float p1 = kv ? tc05::fast_exp2(fmaf(__uint_as_float(sr[2 * j + 1]), c, -m[2 * j + 1])) : 0.f;
        l[2 * j] += p0, l[2 * j + 1] += p1;
        pk[j] = pack_f16(p0, p1);
      }
      if (i > 1) ok = __all_sync(FULL, ok && um::wait_or_abort(&bars.pfree[i & 1], ((i >> 1) - 1) & 1, abort));
      if (ok) {
        uint8_t* row = sP(i) + L * 128;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          *reinterpret_cast<uint4*>(row + ((ch ^ (L & 7)) << 4)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      }
      tc05::fence_proxy_async_smem();
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.pfull[i & 1]);
      if (act) has_act = true;
      else has_vid = true;
      if (!last) continue;

      // ---- segment done: the row sums (while the last P V runs), then O = s_g(V) O_video + O_action
      {
        float v[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = l[q];
        bars.red[wr][lane] = um::reduce_scatter32<false>(v, lane);
      }
      um::softmax_sync();
      float lt[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) lt[q] = (bars.red[0][q] + bars.red[1][q]) + (bars.red[2][q] + bars.red[3][q]);
      um::softmax_sync();
      float o[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) o[q] = 0.f;
      ok = __all_sync(FULL, ok && um::wait_or_abort(&bars.ofull[seg & 1], (seg >> 1) & 1, abort));
      if (ok) {
        tc05::fence_after_sync();
        if (has_vid) {
          uint32_t ov[32];
          tc05::tmem_ld32(o_vid + lane_off, ov);
          tc05::tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = sg_v * __uint_as_float(ov[q]);
        }
        if (has_act) {
          uint32_t oa[32];
          tc05::tmem_ld32(o_act + lane_off, oa);
          tc05::tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] += __uint_as_float(oa[q]);
        }
      }
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.ofree[seg & 1]);
      split_finish_segment(a, tw.b, tw.h, *reinterpret_cast<volatile int*>(&bars.part_k),
                           *reinterpret_cast<volatile int*>(&bars.part_r), L, wr, lane, o, lt, m, &bars.last,
                           sK(0), kStageParts, &bars.mfull, abort);
    }
  } else {
    regs_dec<kRegsConv>();
    // ---------------------------------------------------------------- converters
    // warps 8-11: Q and K tiles; warps 12-15: V tiles.  Warp g of a group decodes row groups g,
    // g + 4, g + 8, g + 12 of a raw tile (decode_rows); in-place bf16 tiles are split by 16-byte
    // chunks over the group's 128 threads.  Every warp of the group arrives on the tile's barriers.
    const bool is_k = warp < 12;
    const int g = warp & 3;
    const int t = 32 * g + lane;
    TileWalk<kKeys> cw;
    cw.init_at(a, part_b, part_h, t0);
    int seg = -1, r = 0;
    int nact[kStages] = {0, 0};
    bool ok = true;
    for (int i = 0; i < n; ++i, cw.next(a)) {
      if (is_k && (i == 0 || cw.t == 0)) {
        ++seg;
        ok = __all_sync(FULL, ok && um::wait_or_abort(&bars.qland[seg & 1], (seg >> 1) & 1, abort));
        if (ok) bf16_tile_to_f16(sQ(seg), kQ, t, 32 * kConvWarps);
        tc05::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.qfull[seg & 1]);
      }
      const int st = i % kStages;
      uint8_t* tile = is_k ? sK(st) : sV(st);
      uint64_t* empty = is_k ? bars.kempty : bars.vempty;
      if (i >= kStages) ok = __all_sync(FULL, ok && um::wait_or_abort(&empty[st], ((i / kStages) - 1) & 1, abort));
      if (cw.t == 0) {
        uint64_t* land = is_k ? bars.kland : bars.vland;
        ok = __all_sync(FULL, ok && um::wait_or_abort(&land[st], nact[st] & 1, abort));
        ++nact[st];
        if (ok) bf16_tile_to_f16(tile, kTile, t, 32 * kConvWarps);
      } else {
        const int sl = r % kRaw;
        uint64_t* full = is_k ? bars.rkfull : bars.rvfull;
        ok = __all_sync(FULL, ok && um::wait_or_abort(&full[sl], (r / kRaw) & 1, abort));
        if (ok) decode_rows(is_k ? rK(sl) : rV(sl), tile, g, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(is_k ? &bars.rkfree[sl] : &bars.rvfree[sl]);
        ++r;
      }
      tc05::fence_proxy_async_smem();  // generic writes to the tile before the MMA reads it
      __syncwarp();
      if (lane == 0) mbar_arrive(is_k ? &bars.kfull[st] : &bars.vfull[st]);
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  tc05::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    mbar_wait(&bars.done, 0);
    tc05::fence_after_sync();
    tc05::tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && bars.abort && a.err) atomicExch(a.err, int(WAM_ERR_TIMEOUT));
}

// Action self-attention of a layer outside the interaction set (no video buffer): one CTA of
// two warps per (episode, head), the n_act <= 32 action keys staged with cp.async into padded
// shared memory rows (272 B pitch: conflict-free ldmatrix), one softmax per row in registers.
constexpr int kSelfPitch = 128 * 2 + 16;

__global__ void __launch_bounds__(64)
action_self_kernel(const __grid_constant__ ActionArgs a) {
  __shared__ __align__(16) uint8_t sm[3][32 * kSelfPitch];
  grid_dependency_wait();  // programmatic dependent launch: inputs ready from here on
  grid_launch_dependents();
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned FULL = 0xffffffffu;
  const __nv_bfloat16* src[3] = {static_cast<const __nv_bfloat16*>(a.qa),
                                 static_cast<const __nv_bfloat16*>(a.ka),
                                 static_cast<const __nv_bfloat16*>(a.va)};
  for (int cidx = tid; cidx < 3 * 32 * 16; cidx += 64) {
    const int ts = cidx >> 9, r = (cidx >> 4) & 31, ch = cidx & 15;
    const int rr = r < a.n_act ? r : 0;  // rows past n_act read nothing and are zero-filled
    const __nv_bfloat16* g = src[ts] + ((int64_t(b) * a.n_act + rr) * a.H + h) * 128 + ch * 8;
    const uint32_t d = smem_u32(&sm[ts][r * kSelfPitch + ch * 16]);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(g),
                 "r"(r < a.n_act ? 16 : 0)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  const int g = lane >> 2, t4 = lane & 3;
  const uint32_t sq = smem_u32(sm[0]), sk = smem_u32(sm[1]), sv = smem_u32(sm[2]);
  // S = Q K^T for this warp's 16 rows x 32 keys
  float s[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    uint32_t qf[4];
    ldsm_x4(sq + (16 * warp + (lane & 15)) * kSelfPitch + (16 * kk + (lane >> 4) * 8) * 2, qf[0],
            qf[1], qf[2], qf[3]);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sk + (16 * p + (lane & 7) + (lane >> 4) * 8) * kSelfPitch + (16 * kk + ((lane >> 3) & 1) * 8) * 2,
              b0, b1, b2, b3);
      mma_bf16(s[2 * p], qf, b0, b1);
      mma_bf16(s[2 * p + 1], qf, b2, b3);
    }
  }
  const float c = a.scale_log2;
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int key = 8 * j + 2 * t4;
    if (key >= a.n_act) s[j][0] = s[j][2] = -INFINITY;
    if (key + 1 >= a.n_act) s[j][1] = s[j][3] = -INFINITY;
    mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
    mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 2));
  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    s[j][0] = ex2(fmaf(s[j][0], c, -mx0 * c));
    s[j][1] = ex2(fmaf(s[j][1], c, -mx0 * c));
    s[j][2] = ex2(fmaf(s[j][2], c, -mx1 * c));
    s[j][3] = ex2(fmaf(s[j][3], c, -mx1 * c));
    l0 += s[j][0] + s[j][1];
    l1 += s[j][2] + s[j][3];
  }
  l0 += __shfl_xor_sync(FULL, l0, 1);
  l0 += __shfl_xor_sync(FULL, l0, 2);
  l1 += __shfl_xor_sync(FULL, l1, 1);
  l1 += __shfl_xor_sync(FULL, l1, 2);
  // O = P V on tf32 tiles, with the same key permutation inside each 8-key group as the
  // fused read (S accumulators are the A fragment, ldmatrix.trans registers the B fragment)
  uint32_t pt[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    pt[j][0] = to_tf32(s[j][0]);
    pt[j][1] = to_tf32(s[j][2]);
    pt[j][2] = to_tf32(s[j][1]);
    pt[j][3] = to_tf32(s[j][3]);
  }
  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
#pragma unroll
  for (int kb16 = 0; kb16 < 2; ++kb16) {
    const int j0 = 2 * kb16, j1 = j0 + 1;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      uint32_t r0, r1, r2, r3;
      ldsm_x4_t(sv + (16 * kb16 + (lane & 7) + ((lane >> 3) & 1) * 8) * kSelfPitch + (16 * p + (lane >> 4) * 8) * 2,
                r0, r1, r2, r3);
      mma_tf32(o[2 * p], pt[j0][0], pt[j0][1], pt[j0][2], pt[j0][3], bf16_lo_bits(r0), bf16_hi_bits(r0));
      mma_tf32(o[2 * p], pt[j1][0], pt[j1][1], pt[j1][2], pt[j1][3], bf16_lo_bits(r1), bf16_hi_bits(r1));
      mma_tf32(o[2 * p + 1], pt[j0][0], pt[j0][1], pt[j0][2], pt[j0][3], bf16_lo_bits(r2), bf16_hi_bits(r2));
      mma_tf32(o[2 * p + 1], pt[j1][0], pt[j1][1], pt[j1][2], pt[j1][3], bf16_lo_bits(r3), bf16_hi_bits(r3));
    }
  }
  const float i0 = 1.f / l0, i1 = 1.f / l1;
  const int r0 = 16 * warp + g, r1 = r0 + 8;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int col = 8 * j + 2 * t4;
    if (r0 < a.n_act) {
      const int64_t off = ((int64_t(b) * a.n_act + r0) * a.H + h) * 128 + col;
      if (a.o_f32) *reinterpret_cast<float2*>(static_cast<float*>(a.o) + off) = make_float2(o[j][0] * i0, o[j][1] * i0);
      else *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(a.o) + off) = pack_bf16(o[j][0] * i0, o[j][1] * i0);
    }
    if (r1 < a.n_act) {
      const int64_t off = ((int64_t(b) * a.n_act + r1) * a.H + h) * 128 + col;
      if (a.o_f32) *reinterpret_cast<float2*>(static_cast<float*>(a.o) + off) = make_float2(o[j][2] * i1, o[j][3] * i1);
      else *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(a.o) + off) = pack_bf16(o[j][2] * i1, o[j][3] * i1);
    }
  }
}

}  // namespace

static int action_bn(const ActionArgs& a) { return a.T % 128 == 0 ? 128 : 64; }

int action_tc_total_tiles(const ActionArgs& a) {
  const int bn = action_bn(a);
  int G = 0;
  for (int b = 0; b < a.B; ++b)
    G += a.H * (1 + (a.with_video ? int(a.fl.nvalid[b]) * (a.T / bn) : 0));
  return G;
}

int action_tc_max_parts(const ActionArgs& a, int P, int G) {
  const int bn = action_bn(a);
  int g = 0, mx = 1;
  for (int b = 0; b < a.B; ++b) {
    const int nb = 1 + (a.with_video ? int(a.fl.nvalid[b]) * (a.T / bn) : 0);
    for (int h = 0; h < a.H; ++h, g += nb) {
      const int lo = int((int64_t(g + 1) * P + G - 1) / G) - 1;
      const int hi = int((int64_t(g + nb) * P + G - 1) / G) - 1;
      if (hi - lo + 1 > mx) mx = hi - lo + 1;
    }
  }
  return mx;
}

int action_aligned_plan(ActionArgs& a, int sms) {
  // part size S video tiles: the smallest that fits every part of every head in one wave of
  // `sms` CTAs (or one part per head when even that does not fit); kparts[b] = ceil(nv_b / S)
  int G = 0, V = 0, max_nv = 1;
  for (int b = 0; b < a.B; ++b) {
    const int nv = a.with_video ? int(a.fl.nvalid[b]) * (a.T / 128) : 0;
    G += a.H * (1 + nv);
    V += a.H * nv;
    max_nv = nv > max_nv ? nv : max_nv;
  }
  int S = sms > 0 ? (V + sms - 1) / sms : max_nv;
  if (S < 1) S = 1;
  for (;; ++S) {
    int64_t total = 0;
    for (int b = 0; b < a.B; ++b) {
      const int nv = a.with_video ? int(a.fl.nvalid[b]) * (a.T / 128) : 0;
      total += int64_t(a.H) * (nv > 0 ? (nv + S - 1) / S : 1);
    }
    if (total <= sms || S >= max_nv) break;
  }
  int P = 0, mx = 1;
  for (int b = 0; b < a.B; ++b) {
    const int nv = a.with_video ? int(a.fl.nvalid[b]) * (a.T / 128) : 0;
    const int k = nv > 0 ? (nv + S - 1) / S : 1;
    a.kparts[b] = uint16_t(k);
    P += a.H * k;
    mx = k > mx ? k : mx;
  }
  a.G = G;
  a.P = P;
  a.max_parts = mx;
  return P;
}

size_t action_tc_workspace_bytes(int BH, int max_parts) {
  if (max_parts <= 1) return 0;
  return kTicketBytes + size_t(BH) * max_parts * kSlotFloats * sizeof(float);
}

// CTAs per (episode, head) of the cluster read: as many as the SMs allow (at most 8, the
// portable cluster size) while all B*H clusters still fit on the GPU at once.  The number of
// co-resident clusters of each size is asked of the runtime once per device.
static int umma_split(int BH, int dev) {
  // Filled and read under one lock, so a second host thread never sees a half-filled table.
  static int max_clusters[32][um::kMaxSplit + 1];
  static bool known[32];
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (!known[dev]) {
    for (int k = 1; k <= um::kMaxSplit; ++k) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(unsigned(k));
      cfg.blockDim = dim3(um::kThreads);
      cfg.dynamicSmemBytes = um::kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = unsigned(k);
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, action_umma_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
      max_clusters[dev][k] = n;
    }
    known[dev] = true;
  }
  for (int k = um::kMaxSplit; k > 1; --k)
    if (max_clusters[dev][k] >= BH) return k;
  return max_clusters[dev][1] > 0 ? 1 : 0;
}

cudaError_t launch_action_nvfp4(const ActionArgs& a, cudaStream_t s) {
  ActionMaps maps;
  if (!make_tmap_bf16(&maps.q, a.qa, a.B, a.n_act, a.H, 32) ||
      !make_tmap_bf16(&maps.ka, a.ka, a.B, a.n_act, a.H, 128) ||
      !make_tmap_bf16(&maps.va, a.va, a.B, a.n_act, a.H, 128))
    return cudaErrorInvalidValue;
  maps.fk = maps.ka, maps.fv = maps.va;  // unused: the video tiles come by bulk copies
  cudaError_t e = cudaFuncSetAttribute(action_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fq::kSmemBytes);
  if (e != cudaSuccess) return e;
  // the warpgroups' register shares add up to exactly the launch allocation: a build that
  // launched with fewer registers per thread would leave the softmax warps' increase unmet
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, action_nvfp4_kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != int(fq::kRegsLaunch)) return cudaErrorInvalidDeviceFunction;
  return launch_pdl(action_nvfp4_kernel, dim3(unsigned(a.P)), dim3(fq::kThreads), fq::kSmemBytes, s, 0, a,
                    maps);
}

cudaError_t launch_action_tc(const ActionArgs& a, cudaStream_t s) {
  if (!a.with_video) {
    return launch_pdl(action_self_kernel, dim3(a.H, a.B), dim3(64), 0, s, 0, a);
  }
  const int bn = action_bn(a);
  const bool umma = bn == 128;
  ActionMaps maps;
  const int N = a.F * a.T;
  if (!make_tmap_bf16(&maps.q, a.qa, a.B, a.n_act, a.H, 32) ||
      !make_tmap_bf16(&maps.ka, a.ka, a.B, a.n_act, a.H, bn) ||
      !make_tmap_bf16(&maps.va, a.va, a.B, a.n_act, a.H, bn))
    return cudaErrorInvalidValue;
  if (a.with_video) {
    if (!make_tmap_bf16(&maps.fk, a.fk, a.B, N, a.H, bn) ||
        !make_tmap_bf16(&maps.fv, a.fv, a.B, N, a.H, bn))
      return cudaErrorInvalidValue;
  } else {
    maps.fk = maps.ka, maps.fv = maps.va;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 32) return cudaErrorInvalidDevice;
  // Set on every call (a host-side attribute write, no device work): nothing cached here can
  // go stale across devices, threads or a device reset.
  cudaError_t e = cudaFuncSetAttribute(action_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(action_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, um::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (umma) {
    ActionArgs ac = a;
    ac.ksplit = umma_split(a.B * a.H, dev);
    if (ac.ksplit < 1) return cudaErrorUnknown;
    return launch_pdl(action_umma_kernel, dim3(unsigned(a.B * a.H * ac.ksplit)), dim3(um::kThreads),
                      um::kSmemBytes, s, unsigned(ac.ksplit), ac, maps);
  }
  // 64-key tiles (T % 128 != 0): the mma.sync kernel
  action_tc_kernel<64><<<a.P, kThreads, kSmemBytes, s>>>(a, maps);
  return cudaGetLastError();
}

}  // namespace wam
