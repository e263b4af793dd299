// Block-causal video prefill on the sm_100a tensor cores (tcgen05.mma, TMEM accumulators,
// TMA-fed shared memory); bf16 inputs, D = 128, T % 128 == 0.
//
// One CTA computes up to 256 query tokens (two 128-row tiles Q0, Q1) of one (episode, frame,
// head) against every key tile the block-causal predicate allows ("Long-WAM: Scaling the
// Context of World-Action Models | Summary" §3.1-3.2); or, when the host pairs the items of a
// one-wave call, the same query tile of two frames of one episode, Q1's keys a prefix of Q0's.  T is a multiple of 128, so every
// 128 x 128 tile is wholly visible or wholly masked: the host work list holds only visible key
// frames and no element mask is applied.  Keys of frames below f_begin come from the layer's
// cache, the others from the call's new K/V.  Each K/V tile loaded feeds both query tiles.
//
// For query tile w and key tile j (128 keys):
//   S_w = Q_w K_j^T           tcgen05.mma, A and B from shared memory -> TMEM
//   P_w = exp2(S_w c - m_w)   softmax warpgroup w; bf16 P written back over S_w in TMEM
//   O_w += P_w V_j            tcgen05.mma, A from TMEM, B (V, MN-major) from shared memory
// The MMA thread alternates the two tiles (P_0 V, next S_0, P_1 V, next S_1, ...), so the
// tensor core works on one tile while the other tile's warpgroup runs its softmax, a single
// pass over S per tile.  A row's reference max m_w is set by its first 32 scores and only
// moves when a later chunk's max exceeds it by more than 2^64; l, O_w and the P already
// written are then rescaled in TMEM.  S_w of key tile j is issued after P_w V_{j-1}, so its
// completion implies O_w is complete up to j-1 and a rescale needs no extra wait.  The
// numerator and denominator share the reference, so the result is exact either way.
//
// Two helper warps store the CTA's own new K/V tokens (those equal to its query tokens) into
// the layer's cache and fold them into the Interval KV-Fusion accumulator ("世界模型之Faster-WAM
// 详解" §3.3) from the call's input while the attention loop runs, so the store and the fold
// never wait on the pipeline and the per-layer cache is never re-read for fusion.
//
// Warps: 0 TMA producer | 1 TMEM allocator + MMA issuer | 2-3 cache store + fusion |
//        4-7 softmax of Q0, 8-11 softmax of Q1 (thread = query row; warp w reads TMEM lanes
//        32 (w % 4) ..).  Every mbarrier wait is bounded; a wait that gives up raises a
//        CTA-wide abort flag, every role drains what it started, TMEM is freed and the
//        device error word is set.
#include "launch.h"
#include "tcgen05.cuh"

namespace wam {
namespace {

constexpr int kBM = 128, kBN = 128;
constexpr int kThreads = 384;
constexpr int kTile = 128 * 128 * 2;  // one Q, K or V tile: two 64-column swizzled halves
constexpr int kHalf = kTile / 2;
constexpr int kKStages = 3, kVStages = 2;
constexpr uint32_t kTmemCols = 512;   // query tile w: S/P at 256 w, O at 256 w + 128
// A row's reference max only moves when a 32-key chunk's sum of p = 2^(s c - m) exceeds this:
// below it every p stays under 2^64, far from fp32 overflow even summed over every key, and
// bf16/fp32 keep their relative precision at any scale.
constexpr float kChunkSumLimit = 18446744073709551616.f;  // 2^64
// Key pairs (of the 16 in a 32-key chunk) whose exponentials run on the FMA pipe
// (exp2_poly2) instead of the special-function unit.
constexpr uint32_t kPolyPairs = 0x0u;
// P to bf16 by integer rounding and a byte permute instead of the conversion instruction.
constexpr bool kPackPermute = false;

struct PrefillMaps {
  CUtensorMap q, kn, vn, kc, vc;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2], o_full[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
  int unit_next;  // next unclaimed unit of the store + fusion pool
};

constexpr int kSmemBytes = 1024 + (2 + kKStages + kVStages) * kTile + int(sizeof(Bars)) + 64;

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < kWaitSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 31u && *abort) return false;
  }
  *abort = 1;
  return false;
}

// acc[0..3] += v[0..3] at the L2, without a round trip (vector reduction, sm_90+).
__device__ __forceinline__ void red_add_v4(float* acc, float a0, float a1, float a2, float a3) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(acc), "f"(a0), "f"(a1), "f"(a2),
               "f"(a3)
               : "memory");
}

// One unit of the cache store + fusion epilogue: 8 consecutive own token rows of the new K or V
// (128 chunks of 8 elements, 4 per lane of one warp; row0_in is the unit's first row in the
// call's input, row0_out in the cache).  The rows are copied into the layer's cache and folded
// into the fusion accumulator: the first layer of an interval writes w x, a middle layer adds
// w x by L2 reductions (nothing to wait for), the last reads the sum and writes the fused bf16
// pair.  4 chunks in flight per lane (8 measured slower).
__device__ __forceinline__ void store_fuse_unit(const PrefillArgs& a, const void* in_base,
                                                void* store_base, float* acc_base,
                                                void* fused_base, int64_t row0_in,
                                                int64_t row0_out, int h, int lane) {
  constexpr int kU = 4;
  const bool need_acc = a.fuse_on && !a.fuse_first && a.fuse_last;
  const bool middle = a.fuse_on && !a.fuse_first && !a.fuse_last;
  uint4 raw[kU];
  float4 p0[kU], p1[kU];
  int64_t off[kU];
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const int c = lane + 32 * u, r = c >> 4, cc = (c & 15) * 8;
    raw[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(in_base) +
                                             ((row0_in + r) * a.H + h) * 128 + cc);
    off[u] = ((row0_out + r) * a.H + h) * 128 + cc;
    if (need_acc) {
      p0[u] = *reinterpret_cast<const float4*>(acc_base + off[u]);
      p1[u] = *reinterpret_cast<const float4*>(acc_base + off[u] + 4);
    }
  }
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    if (store_base)
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(store_base) + off[u]) = raw[u];
    if (!a.fuse_on) continue;
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&raw[u]);
    float s[8];
    if (need_acc) {
      const float p[8] = {p0[u].x, p0[u].y, p0[u].z, p0[u].w, p1[u].x, p1[u].y, p1[u].z, p1[u].w};
#pragma unroll
      for (int j = 0; j < 8; ++j) s[j] = fmaf(a.fuse_w, __bfloat162float(x[j]), p[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) s[j] = a.fuse_w * __bfloat162float(x[j]);
    }
    if (middle) {
      red_add_v4(acc_base + off[u], s[0], s[1], s[2], s[3]);
      red_add_v4(acc_base + off[u] + 4, s[4], s[5], s[6], s[7]);
    } else if (a.fuse_last) {
      uint4 v;
      v.x = pack_bf16(s[0], s[1]), v.y = pack_bf16(s[2], s[3]);
      v.z = pack_bf16(s[4], s[5]), v.w = pack_bf16(s[6], s[7]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(fused_base) + off[u]) = v;
    } else {
      *reinterpret_cast<float4*>(acc_base + off[u]) = make_float4(s[0], s[1], s[2], s[3]);
      *reinterpret_cast<float4*>(acc_base + off[u] + 4) = make_float4(s[4], s[5], s[6], s[7]);
    }
  }
}

// The CTA's store + fusion work as a pool of units (K units first, then V), claimed one at a
// time through a shared-memory counter by whole warps: the helper warps from the start, each
// softmax warp once its output is written, so a CTA with few key tiles does not wait on two
// warps for its epilogue.  `rows` (a multiple of 8) own tokens from row_in / row_out.
__device__ __forceinline__ void store_fuse_pool(const PrefillArgs& a, int* next, int rows,
                                                int64_t row_in, int64_t row_out, int h,
                                                int lane) {
  if (a.k_store == nullptr && !a.fuse_on) return;
  const int per = rows / 8;
  for (;;) {
    int u = 0;
    if (lane == 0) u = atomicAdd(next, 1);
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u >= 2 * per) break;
    if (u < per)
      store_fuse_unit(a, a.k_new, a.k_store, a.acc_k, a.fused_k, row_in + 8 * u,
                      row_out + 8 * u, h, lane);
    else
      store_fuse_unit(a, a.v_new, a.v_store, a.acc_v, a.fused_v, row_in + 8 * (u - per),
                      row_out + 8 * (u - per), h, lane);
  }
}
// The same for a cross-frame pair: the rows of the two query tiles are not contiguous.
__device__ __forceinline__ void store_fuse_pool_pair(const PrefillArgs& a, int* next,
                                                     int64_t in0, int64_t in1, int64_t out0,
                                                     int64_t out1, int h, int lane) {
  if (a.k_store == nullptr && !a.fuse_on) return;
  constexpr int kPerTile = kBM / 8;  // units of one query tile's rows, of K or of V
  const int per = 2 * kPerTile;
  for (;;) {
    int u = 0;
    if (lane == 0) u = atomicAdd(next, 1);
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u >= 2 * per) break;
    const bool is_v = u >= per;
    const int uu = is_v ? u - per : u, r0 = 8 * (uu % kPerTile);
    const bool t1 = uu >= kPerTile;  // rows of query tile 1
    const int64_t ri = (t1 ? in1 : in0) + r0, ro = (t1 ? out1 : out0) + r0;
    if (!is_v)
      store_fuse_unit(a, a.k_new, a.k_store, a.acc_k, a.fused_k, ri, ro, h, lane);
    else
      store_fuse_unit(a, a.v_new, a.v_store, a.acc_v, a.fused_v, ri, ro, h, lane);
  }
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic)
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^y for a pair on the FMA pipe.  Cody-Waite style range reduction: y = n + f with
// n = round(y) taken from the low mantissa bits of y + 1.5 * 2^23 and f in [-1/2, 1/2]; 2^f by
// a cubic fitted for minimax relative error on that interval (coefficients computed for this
// file with a Remez exchange; max relative error 7.5e-5, below bf16's 2^-9 rounding of P); the
// integer n is then added into the exponent field.  y is clamped to [-126, 127] so the
// exponent stays in range: below -126 the result is 2^-126 instead of ~0, negligible against
// a row sum >= 1.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t y2) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  float y0, y1;
  f2unpack(y2, y0, y1);
  y0 = fminf(fmaxf(y0, -126.f), 127.f);
  y1 = fminf(fmaxf(y1, -126.f), 127.f);
  const uint64_t yc = f2pack(y0, y1);
  const uint64_t t = f2add(yc, f2pack(kRound, kRound));
  const uint64_t f = f2sub(yc, f2sub(t, f2pack(kRound, kRound)));
  uint64_t q = f2fma(f2pack(0.0551716685f, 0.0551716685f), f, f2pack(0.2426111251f, 0.2426111251f));
  q = f2fma(q, f, f2pack(0.6932609677f, 0.6932609677f));
  q = f2fma(q, f, f2pack(0.9999280572f, 0.9999280572f));
  float t0, t1, q0, q1;
  f2unpack(t, t0, t1);
  f2unpack(q, q0, q1);
  return f2pack(__uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23)),
                __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23)));
}

// Two non-negative finite floats to a bf16 pair (first in the low half), rounded to nearest
// (ties away from zero).
__device__ __forceinline__ uint32_t pack_p(float p0, float p1) {
  if (kPackPermute) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(r) : "r"(__float_as_uint(p0) + 0x8000u),
        "r"(__float_as_uint(p1) + 0x8000u));
    return r;
  }
  return pack_bf16(p0, p1);
}



// kPaired: the call's items are cross-frame pairs (a.fl.paired); a separate instantiation, so
// that the per-tile key counts and token offsets of a pair cost nothing in unpaired calls.
template <bool kPaired>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ PrefillMaps maps) {
  // the tensor maps' descriptors first, hidden behind the set-up below (parameter space: the
  // previous kernel on the stream cannot write it)
  if (threadIdx.x == 0) {
    prefetch_tmap(&maps.q), prefetch_tmap(&maps.kn), prefetch_tmap(&maps.vn);
    prefetch_tmap(&maps.kc), prefetch_tmap(&maps.vc);
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align1024(smem_raw);
  // Tiles by arithmetic, not through pointer arrays (a runtime index would put those in local memory).
  auto sQ = [&](int w) { return base + w * kTile; };
  auto sK = [&](int i) { return base + (2 + i) * kTile; };
  auto sV = [&](int i) { return base + (2 + kKStages + i) * kTile; };
  Bars& bars = *reinterpret_cast<Bars*>(base + (2 + kKStages + kVStages) * kTile);
  volatile int* abort = &bars.abort;

  // ---- work item: query tiles 2 qp and 2 qp + 1 of frame f (the second may not exist), or,
  // with a.fl.paired, query tile qt of both frames of the item pair (2 i, 2 i + 1) of one
  // episode: the first reads nk_0 key frames, the second nk_1 <= nk_0, the first nk_1 of the
  // same list, so every key tile loaded feeds both tiles until the second one's keys end.
  const int QT = a.T / kBM, QP = (QT + 1) / 2;
  const int h = int(blockIdx.x % a.H);
  const int rest = int(blockIdx.x / a.H);
  const int tpf = a.T / kBN;
  // (scalars per query tile, selected by w: no local-memory arrays)
  int b, f0, f1, nk0, nk1, qt0, qt1, nq;
  if constexpr (kPaired) {
    const uint32_t i0 = a.fl.item[2 * (rest / QT)], i1 = a.fl.item[2 * (rest / QT) + 1];
    b = item_b(i0);
    f0 = item_f(i0), f1 = item_f(i1);
    nk0 = item_nk(i0), nk1 = item_nk(i1);
    qt0 = qt1 = rest % QT;
    nq = 2;
  } else {
    const int qp = rest % QP;
    const uint32_t it = a.fl.item[rest / QP];
    b = item_b(it);
    f0 = f1 = item_f(it);
    nk0 = nk1 = item_nk(it);
    qt0 = 2 * qp, qt1 = 2 * qp + 1;
    nq = (2 * qp + 1 < QT) ? 2 : 1;                     // query tiles in this CTA
  }
  const int n = nk0 * tpf;                              // key tiles (of the first query tile)
  // key tiles of query tile w, and its first token among the call's query tokens
  auto nw = [&](int w) {
    if constexpr (kPaired) return (w ? nk1 : nk0) * tpf;
    else return n;
  };
  auto qtokw = [&](int w) {
    if constexpr (kPaired) return ((w ? f1 : f0) - a.f_begin) * a.T + (w ? qt1 : qt0) * kBM;
    else return (f0 - a.f_begin) * a.T + (qt0 + w) * kBM;
  };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  auto key_tile = [&](int j, bool& old, int& tok) {
    const int fk = a.fl.vlist[b * a.F + j / tpf], jj = j % tpf;
    old = fk < a.f_begin;
    tok = (old ? fk : fk - a.f_begin) * a.T + jj * kBN;
  };

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);  // MMA completion
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars.s_full[w], 1);
      mbar_init(&bars.p_full[w], 4);
      mbar_init(&bars.o_full[w], 1);
    }
    mbar_init(&bars.done, 1);
    bars.abort = 0;
    bars.unit_next = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc05::tmem_alloc(&bars.tmem_base, kTmemCols);
    tc05::tmem_relinquish();
  }
  tc05::fence_before_sync();
  __syncthreads();
  tc05::fence_after_sync();
  const uint32_t tmem = bars.tmem_base;
  // Up to here only this CTA's shared and tensor memory was touched: the previous kernel on
  // the stream may still be finishing (programmatic dependent launch).
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int k_issued = 0, v_issued = 0;
      mbar_arrive_expect_tx(&bars.q_full, nq * kTile);
      for (int w = 0; w < nq; ++w) {
        tma_load_4d(sQ(w), &maps.q, &bars.q_full, 0, h, qtokw(w), b);
        tma_load_4d(sQ(w) + kHalf, &maps.q, &bars.q_full, 64, h, qtokw(w), b);
      }
      for (int j = 0; j < n; ++j) {
        bool old;
        int tok;
        key_tile(j, old, tok);
        const int ks = j % kKStages, vs = j % kVStages;
        if (j >= kKStages && !wait_bar(&bars.k_empty[ks], ((j / kKStages) - 1) & 1, abort)) break;
        const CUtensorMap* mk = old ? &maps.kc : &maps.kn;
        mbar_arrive_expect_tx(&bars.k_full[ks], kTile);
        tma_load_4d(sK(ks), mk, &bars.k_full[ks], 0, h, tok, b);
        tma_load_4d(sK(ks) + kHalf, mk, &bars.k_full[ks], 64, h, tok, b);
        k_issued = j + 1;
        if (j >= kVStages && !wait_bar(&bars.v_empty[vs], ((j / kVStages) - 1) & 1, abort)) break;
        const CUtensorMap* mv = old ? &maps.vc : &maps.vn;
        mbar_arrive_expect_tx(&bars.v_full[vs], kTile);
        tma_load_4d(sV(vs), mv, &bars.v_full[vs], 0, h, tok, b);
        tma_load_4d(sV(vs) + kHalf, mv, &bars.v_full[vs], 64, h, tok, b);
        v_issued = j + 1;
      }
      // Drain: loads issued must land before the CTA leaves (matters only after an abort).
      for (int j = (k_issued > kKStages ? k_issued - kKStages : 0); j < k_issued; ++j)
        mbar_wait(&bars.k_full[j % kKStages], (j / kKStages) & 1);
      for (int j = (v_issued > kVStages ? v_issued - kVStages : 0); j < v_issued; ++j)
        mbar_wait(&bars.v_full[j % kVStages], (j / kVStages) & 1);
      mbar_wait(&bars.q_full, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = tc05::idesc_bf16_f32(128, 128, false);
      const uint32_t idO = tc05::idesc_bf16_f32(128, 128, true);
      const uint32_t tS[2] = {tmem, tmem + 256}, tO[2] = {tmem + 128, tmem + 384};
      auto issue_S = [&](int w, int j) {
        const uint32_t q_s = smem_u32(sQ(w)), k_s = smem_u32(sK(j % kKStages));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          tc05::mma_ss(tS[w], tc05::smem_desc_sw128(q_s + off, 16, 1024),
                       tc05::smem_desc_sw128(k_s + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_PV = [&](int w, int j) {
        const uint32_t v_s = smem_u32(sV(j % kVStages));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc05::mma_ts(tO[w], tS[w] + 8 * kk, tc05::smem_desc_sw128(v_s + kk * 2048, kHalf, 1024), idO,
                 (j > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = wait_bar(&bars.q_full, 0, abort) && wait_bar(&bars.k_full[0], 0, abort);
      if (ok) {
        tc05::fence_after_sync();
        for (int w = 0; w < nq; ++w) {
          issue_S(w, 0);
          tc05::mma_commit(&bars.s_full[w]);
        }
        tc05::mma_commit(&bars.k_empty[0]);
      }
      for (int j = 0; ok && j < n; ++j) {
        const bool more = j + 1 < n;
        if (!wait_bar(&bars.v_full[j % kVStages], (j / kVStages) & 1, abort)) break;
        if (more && !wait_bar(&bars.k_full[(j + 1) % kKStages], ((j + 1) / kKStages) & 1, abort)) break;
        bool fail = false;
        for (int w = 0; w < nq; ++w) {
          if (j >= nw(w)) continue;  // this query tile's keys have ended
          if (!wait_bar(&bars.p_full[w], j & 1, abort)) { fail = true; break; }
          tc05::fence_after_sync();
          issue_PV(w, j);
          if (j == nw(w) - 1) tc05::mma_commit(&bars.o_full[w]);
          if (j + 1 < nw(w)) {
            issue_S(w, j + 1);
            tc05::mma_commit(&bars.s_full[w]);
          }
        }
        if (fail) break;
        tc05::mma_commit(&bars.v_empty[j % kVStages]);
        if (more) tc05::mma_commit(&bars.k_empty[(j + 1) % kKStages]);
      }
      tc05::mma_commit(&bars.done);  // arrives once every MMA issued above has completed
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax, one row per thread
    // tcgen05.ld / tcgen05.st are warp-collective: every decision in front of one is voted
    // across the warp, so all 32 lanes always execute them together.
    const unsigned FULL = 0xffffffffu;
    const int w = (warp - 4) >> 2;  // query tile of this warpgroup
    if (w < nq) {
      const int r = 32 * (warp & 3) + lane;
      const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
      const uint32_t tS = tmem + 256 * w + lane_off, tO = tmem + 256 * w + 128 + lane_off;
      const float c = a.scale_log2;
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      const int n_own = nw(w);
      for (int j = 0; j < n_own; ++j) {
        ok = __all_sync(FULL, ok && wait_bar(&bars.s_full[w], j & 1, abort));
        if (!ok) continue;
        tc05::fence_after_sync();
        // One pass over S in four 32-column chunks (two per TMEM wait).  P of chunk q goes to
        // TMEM columns [16 q, 16 q + 16), all already read.  Each chunk is first exponentiated
        // against the row's current reference m_ref.  A lane whose chunk sum exceeds 2^64 (or
        // is inf: the first chunk of a row always is, m_ref starts at -inf) moves its reference
        // to the chunk max; l, O (key tiles < j) and the P chunks already written are then
        // scaled by alpha = 2^(m_ref - m_new) and the chunk is redone on the special-function
        // unit.  Lanes that keep their reference scale by 1 (exact), so every TMEM access is
        // warp-collective.
        const uint64_t c2 = f2pack(c, c);
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t x[2][32];
          tc05::tmem_ld32(tS + 64 * q2, x[0]);
          tc05::tmem_ld32(tS + 64 * q2 + 32, x[1]);
          tc05::tmem_wait_ld();
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int q = 2 * q2 + h2;
            uint32_t pk[16];
            uint64_t acc[4] = {0, 0, 0, 0};
            const uint64_t nm2 = f2pack(-m_ref, -m_ref);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint64_t y = f2fma(f2pack(__uint_as_float(x[h2][2 * i]), __uint_as_float(x[h2][2 * i + 1])), c2, nm2);
              uint64_t p;
              if ((kPolyPairs >> i) & 1u) {
                p = exp2_poly2(y);
              } else {
                float y0, y1;
                f2unpack(y, y0, y1);
                p = f2pack(tc05::fast_exp2(y0), tc05::fast_exp2(y1));
              }
              acc[i & 3] = f2add(acc[i & 3], p);
              float p0, p1;
              f2unpack(p, p0, p1);
              pk[i] = pack_p(p0, p1);  // key 2i in the low half
            }
            float s0, s1;
            f2unpack(f2add(f2add(acc[0], acc[1]), f2add(acc[2], acc[3])), s0, s1);
            float csum = s0 + s1;
            const bool up = !(csum <= kChunkSumLimit);
            if (__any_sync(FULL, up)) {
              float cm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
              for (int i = 0; i < 32; i += 2)
                cm[(i >> 1) & 3] = fmaxf(cm[(i >> 1) & 3], fmaxf(__uint_as_float(x[h2][i]), __uint_as_float(x[h2][i + 1])));
              const float m_c = fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3])) * c;
              const float m_new = up ? m_c : m_ref;
              const float alpha = up ? tc05::fast_exp2(m_ref - m_new) : 1.f;
              l *= alpha;
              if (j > 0) {  // O holds P V of key tiles < j (S_w of tile j followed P_w V_{j-1})
#pragma unroll
                for (int qo = 0; qo < 4; ++qo) {
                  uint32_t o[32];
                  tc05::tmem_ld32(tO + 32 * qo, o);
                  tc05::tmem_wait_ld();
#pragma unroll
                  for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                  tc05::tmem_st32(tO + 32 * qo, o);
                }
              }
              for (int qp2 = 0; qp2 < q; ++qp2) {  // P chunks of this tile already written
                uint32_t pw[16];
                tc05::tmem_ld16(tS + 16 * qp2, pw);
                tc05::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&pw[i]);
                  pw[i] = pack_p(__low2float(v) * alpha, __high2float(v) * alpha);
                }
                tc05::tmem_st16(tS + 16 * qp2, pw);
              }
              tc05::tmem_wait_st();
              m_ref = m_new;
              csum = 0.f;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float p0 = tc05::fast_exp2(fmaf(__uint_as_float(x[h2][2 * i]), c, -m_ref));
                const float p1 = tc05::fast_exp2(fmaf(__uint_as_float(x[h2][2 * i + 1]), c, -m_ref));
                csum += p0 + p1;
                pk[i] = pack_p(p0, p1);
              }
            }
            l += csum;
            tc05::tmem_st16(tS + 16 * q, pk);
          }
        }
        tc05::tmem_wait_st();
        tc05::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[w]);
      }
      // epilogue: O / l to global memory
      ok = __all_sync(FULL, ok && wait_bar(&bars.o_full[w], 0, abort));
      if (ok) {
        tc05::fence_after_sync();
        const float inv = 1.f / l;
        const int64_t qtok = int64_t(a.f_end - a.f_begin) * a.T;
        const int64_t row = int64_t(b) * qtok + qtokw(w) + r;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tc05::tmem_ld32(tO + 32 * q, o);
          tc05::tmem_wait_ld();
          const int64_t off = (row * a.H + h) * 128 + 32 * q;
          if (a.o_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.o) + off);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                   __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + off);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 u;
              u.x = pack_bf16(__uint_as_float(o[8 * i]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
              u.y = pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
              u.z = pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
              u.w = pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
              dst[i] = u;
            }
          }
        }
      }
    }
  }
  if (warp >= 2) {
    // ------------------------------------------------------------ cache store + fusion
    // The CTA's own tokens, read from the call's new K/V: the helper warps start at once, while
    // the attention loop runs; each softmax warp joins once its output is written (converged:
    // every branch in the softmax is warp-uniform).
    // first own token row of query tile w in the call's new K/V and in the layer's cache
    const int64_t in0 = int64_t(b) * (int64_t(a.f_end - a.f_begin) * a.T);
    const int64_t out0 = int64_t(b) * (int64_t(a.F) * a.T);
    if constexpr (kPaired)
      store_fuse_pool_pair(a, &bars.unit_next, in0 + qtokw(0), in0 + qtokw(1),
                           out0 + int64_t(f0) * a.T + qt0 * kBM, out0 + int64_t(f1) * a.T + qt1 * kBM, h, lane);
    else
      store_fuse_pool(a, &bars.unit_next, nq * kBM, in0 + qtokw(0), out0 + int64_t(f0) * a.T + qt0 * kBM, h,
                      lane);
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();  // reconverge the single-lane roles with the rest of their warp
  tc05::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    mbar_wait(&bars.done, 0);  // every MMA has completed (bounded)
    tc05::fence_after_sync();
    tc05::tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && bars.abort && a.err) atomicExch(a.err, int(WAM_ERR_TIMEOUT));
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
  // Set on every call (a host-side attribute write, no device work): nothing cached here can
  // go stale across devices, threads or a device reset.
  cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int QT = a.T / kBM, QP = (QT + 1) / 2;
  const int64_t grid = a.fl.paired ? int64_t(a.fl.n_items / 2) * QT * a.H : int64_t(a.fl.n_items) * QP * a.H;
  if (a.fl.paired)
    return launch_pdl(prefill_tc_kernel<true>, dim3(unsigned(grid)), dim3(kThreads), kSmemBytes, s, 0, a, maps);
  return launch_pdl(prefill_tc_kernel<false>, dim3(unsigned(grid)), dim3(kThreads), kSmemBytes, s, 0, a, maps);
}

}  // namespace wam
