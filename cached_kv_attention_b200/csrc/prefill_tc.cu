// Block-causal video prefill on the sm_100a tensor cores (tcgen05.mma, TMEM accumulators,
// TMA-fed shared memory); bf16 inputs, D = 128, T % 128 == 0.
//
// One CTA computes 128 query tokens of one (episode, frame, head) against every key tile the
// block-causal predicate allows ("Long-WAM: Scaling the Context of World-Action Models |
// Summary" §3.1-3.2).  T is a multiple of 128, so every 128 x 128 tile is wholly visible or
// wholly masked: the host work list holds only the visible key frames and no element mask is
// applied.  Keys of frames below f_begin come from the layer's cache, the others from the
// call's new K/V.
//
// Per key tile j (128 keys):   S_j = Q K_j^T          tcgen05.mma -> TMEM (two S buffers)
//                              P_j = exp2(S_j c - m)   softmax warps, bf16 -> shared memory
//                              O  += P_j V_j           tcgen05.mma -> TMEM (one O buffer)
// The MMA thread issues S_{j+1} before P_j V_j, so the tensor core computes the next scores
// while the softmax warps work on the current ones.  The reference max m of a row only moves
// when a tile raises the row max by more than 8 (a factor 2^8); O and l are then rescaled in
// TMEM, which needs P_{j-1} V_{j-1} to have landed.  Otherwise p stays below 2^8 and nothing
// is rescaled (exact arithmetic either way: numerator and denominator share the reference).
//
// While the CTA's own 128 tokens of K/V are resident, two helper warps store them into the
// layer's cache and fold them into the Interval KV-Fusion accumulator ("世界模型之Faster-WAM
// 详解" §3.3), so the per-layer K/V is never re-read for fusion.
//
// Warps: 0 TMA producer | 1 TMEM allocator + MMA issuer | 2-3 cache store and fusion |
//        4-7 softmax (thread = query row; warp w reads TMEM lanes 32 (w % 4) ..).
// Every mbarrier wait is bounded; a wait that gives up raises a CTA-wide abort flag, every
// role drains what it started, TMEM is freed and the device error word is set.
#include "launch.h"
#include "tcgen05.cuh"

namespace wam {
namespace {

constexpr int kBM = 128, kBN = 128;
constexpr int kThreads = 256;
constexpr int kTile = 128 * 128 * 2;  // one Q, K, V or P tile: two 64-column swizzled halves
constexpr int kHalf = kTile / 2;
constexpr uint32_t kTmemCols = 512;   // S0 [0,128) S1 [128,256) O [256,384)
constexpr float kRescaleLog2 = 8.f;

struct PrefillMaps {
  CUtensorMap q, kn, vn, kc, vc;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], s_free[2], p_full[2], p_empty[2];
  uint64_t o_full, done;
  uint32_t tmem_base;
  int abort;
};

constexpr int kSmemBytes = 1024 + 7 * kTile + int(sizeof(Bars)) + 64;

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < kWaitSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 31u && *abort) return false;
  }
  *abort = 1;
  return false;
}

// Store (and fold into the fusion accumulator) one resident 128-token K or V tile; 64 threads.
// Each thread handles 4 chunks of 8 elements per round and issues all their accumulator loads
// before using any of them, so the read-modify-write keeps several loads in flight.
__device__ __forceinline__ void store_fuse_tile128(const PrefillArgs& a, const uint8_t* tile,
                                                   void* store_base, float* acc_base,
                                                   void* fused_base, int64_t row0, int h, int t) {
  constexpr int kU = 4;
  for (int c0 = t; c0 < kBN * 16; c0 += 64 * kU) {
    uint4 raw[kU];
    float4 p0[kU], p1[kU];
    int64_t off[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + 64 * u, r = c >> 4, cc = (c & 15) * 8;
      raw[u] = *reinterpret_cast<const uint4*>(tile + swz128<kBN>(r, cc));
      off[u] = ((row0 + r) * a.H + h) * 128 + cc;
      if (a.fuse_on && !a.fuse_first) {
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
      if (a.fuse_first) {
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] = a.fuse_w * __bfloat162float(x[j]);
      } else {
        const float p[8] = {p0[u].x, p0[u].y, p0[u].z, p0[u].w, p1[u].x, p1[u].y, p1[u].z, p1[u].w};
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] = fmaf(a.fuse_w, __bfloat162float(x[j]), p[j]);
      }
      if (a.fuse_last) {
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
}

// Pulls the accumulator rows of the CTA's own 128 tokens into L2 ahead of the fold (64 threads).
__device__ __forceinline__ void prefetch_acc_rows(const PrefillArgs& a, const float* acc, int64_t row0,
                                                  int h, int t) {
  for (int r = t; r < kBN; r += 64) {
    const float* p = acc + ((row0 + r) * a.H + h) * 128;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], 512;" ::"l"(p) : "memory");
  }
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ PrefillArgs a, const __grid_constant__ PrefillMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK[2] = {base + kTile, base + 2 * kTile};
  uint8_t* sV[2] = {base + 3 * kTile, base + 4 * kTile};
  uint8_t* sP[2] = {base + 5 * kTile, base + 6 * kTile};
  Bars& bars = *reinterpret_cast<Bars*>(base + 7 * kTile);
  volatile int* abort = &bars.abort;

  const int QT = a.T / kBM;
  const int h = int(blockIdx.x % a.H);
  const int rest = int(blockIdx.x / a.H);
  const int qt = rest % QT;
  const uint32_t it = a.fl.item[rest / QT];
  const int b = item_b(it), f = item_f(it), nk = item_nk(it);
  const int tpf = a.T / kBN;
  const int n = nk * tpf;                              // key tiles
  const int qtok0 = (f - a.f_begin) * a.T + qt * kBM;  // first query row of the call
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.k_empty[s], 2);  // MMA completion + store warps
      mbar_init(&bars.v_empty[s], 2);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.s_free[s], 4);
      mbar_init(&bars.p_full[s], 4);
      mbar_init(&bars.p_empty[s], 1);
    }
    mbar_init(&bars.o_full, 1);
    mbar_init(&bars.done, 1);
    bars.abort = 0;
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
  const uint32_t tS[2] = {tmem, tmem + 128};
  const uint32_t tO = tmem + 256;

  // Key tiles in list order, except that the CTA's own tile (its own 128 tokens) is swapped to
  // the end: the store warps then hold its K/V stage while no later tile needs that stage.
  int own_u = nk - 1;  // position of the query frame among the visible frames
  for (int u = 0; u < nk; ++u)
    if (a.fl.vlist[b * a.F + u] == f) own_u = u;
  const int own_j = own_u * tpf + qt;
  auto key_tile = [&](int j, bool& old, int& tok, int& fk, int& jj) {
    const int jm = j == n - 1 ? own_j : (j == own_j ? n - 1 : j);
    fk = a.fl.vlist[b * a.F + jm / tpf];
    jj = jm % tpf;
    old = fk < a.f_begin;
    tok = (old ? fk : fk - a.f_begin) * a.T + jj * kBN;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      mbar_arrive_expect_tx(&bars.q_full, kTile);
      tma_load_4d(sQ, &maps.q, &bars.q_full, 0, h, qtok0, b);
      tma_load_4d(sQ + kHalf, &maps.q, &bars.q_full, 64, h, qtok0, b);
      for (int j = 0; j < n; ++j) {
        const int s = j & 1;
        bool old;
        int tok, fk, jj;
        key_tile(j, old, tok, fk, jj);
        const CUtensorMap* mk = old ? &maps.kc : &maps.kn;
        const CUtensorMap* mv = old ? &maps.vc : &maps.vn;
        if (j >= 2 && !wait_bar(&bars.k_empty[s], ((j >> 1) - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&bars.k_full[s], kTile);
        tma_load_4d(sK[s], mk, &bars.k_full[s], 0, h, tok, b);
        tma_load_4d(sK[s] + kHalf, mk, &bars.k_full[s], 64, h, tok, b);
        if (j >= 2 && !wait_bar(&bars.v_empty[s], ((j >> 1) - 1) & 1, abort)) {
          issued = -(j + 1);  // K_j issued, V_j not
          break;
        }
        mbar_arrive_expect_tx(&bars.v_full[s], kTile);
        tma_load_4d(sV[s], mv, &bars.v_full[s], 0, h, tok, b);
        tma_load_4d(sV[s] + kHalf, mv, &bars.v_full[s], 64, h, tok, b);
        issued = j + 1;
      }
      // Drain: loads issued must land before the CTA leaves (matters only after an abort).
      const int nk_issued = issued < 0 ? -issued : issued;
      const int nv_issued = issued < 0 ? -issued - 1 : issued;
      for (int j = (nk_issued > 2 ? nk_issued - 2 : 0); j < nk_issued; ++j)
        mbar_wait(&bars.k_full[j & 1], (j >> 1) & 1);
      for (int j = (nv_issued > 2 ? nv_issued - 2 : 0); j < nv_issued; ++j)
        mbar_wait(&bars.v_full[j & 1], (j >> 1) & 1);
      mbar_wait(&bars.q_full, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = tc05::idesc_bf16_f32(128, 128, false);
      const uint32_t idO = tc05::idesc_bf16_f32(128, 128, true);
      const uint32_t q_s = smem_u32(sQ);
      bool ok = wait_bar(&bars.q_full, 0, abort);
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int s = j & 1;
          if (!wait_bar(&bars.k_full[s], (j >> 1) & 1, abort)) break;
          if (j >= 2 && !wait_bar(&bars.s_free[s], ((j >> 1) - 1) & 1, abort)) break;
          tc05::fence_after_sync();
          const uint32_t k_s = smem_u32(sK[s]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            tc05::mma_ss(tS[s], tc05::smem_desc_sw128(q_s + off, 16, 1024),
                         tc05::smem_desc_sw128(k_s + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
          }
          tc05::mma_commit(&bars.k_empty[s]);
          tc05::mma_commit(&bars.s_full[s]);
        }
        if (j >= 1) {
          const int jp = j - 1, sp = jp & 1;
          if (!wait_bar(&bars.v_full[sp], (jp >> 1) & 1, abort)) break;
          if (!wait_bar(&bars.p_full[sp], (jp >> 1) & 1, abort)) break;
          tc05::fence_after_sync();
          const uint32_t p_s = smem_u32(sP[sp]), v_s = smem_u32(sV[sp]);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t poff = (kk >> 2) * kHalf + (kk & 3) * 32;
            tc05::mma_ss(tO, tc05::smem_desc_sw128(p_s + poff, 16, 1024),
                         tc05::smem_desc_sw128(v_s + kk * 2048, kHalf, 1024), idO,
                         (jp > 0 || kk > 0) ? 1u : 0u);
          }
          tc05::mma_commit(&bars.v_empty[sp]);
          tc05::mma_commit(&bars.p_empty[sp]);
          if (jp == n - 1) tc05::mma_commit(&bars.o_full);
        }
      }
      tc05::mma_commit(&bars.done);  // arrives once every MMA issued above has completed
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ cache store + fusion
    // The 64 threads run every iteration (a failed wait skips work, never the named barrier).
    const int t = threadIdx.x - 64;
    const bool do_store = a.k_store != nullptr || a.fuse_on;
    const int64_t N = int64_t(a.F) * a.T;
    if (a.fuse_on && !a.fuse_first) {
      const int64_t own_row0 = int64_t(b) * N + int64_t(f) * a.T + qt * kBN;
      prefetch_acc_rows(a, a.acc_k, own_row0, h, t);
      prefetch_acc_rows(a, a.acc_v, own_row0, h, t);
    }
    for (int j = 0; j < n; ++j) {
      const int s = j & 1;
      bool old;
      int tok, fk, jj;
      key_tile(j, old, tok, fk, jj);
      const bool own = do_store && fk == f && jj == qt;
      const int64_t row0 = int64_t(b) * N + int64_t(f) * a.T + jj * kBN;
      const bool okk = wait_bar(&bars.k_full[s], (j >> 1) & 1, abort);
      if (okk && own) store_fuse_tile128(a, sK[s], a.k_store, a.acc_k, a.fused_k, row0, h, t);
      asm volatile("bar.sync 2, 64;" ::: "memory");
      if (t == 0 && okk) mbar_arrive(&bars.k_empty[s]);
      const bool okv = wait_bar(&bars.v_full[s], (j >> 1) & 1, abort);
      if (okv && own) store_fuse_tile128(a, sV[s], a.v_store, a.acc_v, a.fused_v, row0, h, t);
      asm volatile("bar.sync 2, 64;" ::: "memory");
      if (t == 0 && okv) mbar_arrive(&bars.v_empty[s]);
    }
  } else {
    // ------------------------------------------------------------ softmax, one row per thread
    // tcgen05.ld / tcgen05.st are warp-collective: every decision in front of one is voted
    // across the warp, so all 32 lanes always execute them together.
    const unsigned FULL = 0xffffffffu;
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const float c = a.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int s = j & 1;
      ok = __all_sync(FULL, ok && wait_bar(&bars.s_full[s], (j >> 1) & 1, abort));
      if (!ok) continue;
      tc05::fence_after_sync();
      uint32_t x[4][32];
#pragma unroll
      for (int q = 0; q < 4; ++q) tc05::tmem_ld32(tS[s] + lane_off + 32 * q, x[q]);
      tc05::tmem_wait_ld();
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_free[s]);
      // row max and row sum over 8 independent accumulators (short dependency chains)
      float mx8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < 32; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], __uint_as_float(x[q][i]));
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_cand = mx * c;
      bool rescale = false;
      float alpha = 1.f;
      if (j == 0) {
        m_ref = m_cand;
      } else if (m_cand > m_ref + kRescaleLog2) {
        alpha = exp2f(m_ref - m_cand);
        l *= alpha;
        m_ref = m_cand;
        rescale = true;
      }
      float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p = tc05::fast_exp2(fmaf(__uint_as_float(x[q][i]), c, -m_ref));
          sum8[i & 7] += p;
          x[q][i] = __float_as_uint(p);
        }
      l += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
      // P buffer s is free once P_{j-2} V_{j-2} has completed
      if (j >= 2) {
        ok = __all_sync(FULL, wait_bar(&bars.p_empty[s], ((j >> 1) - 1) & 1, abort));
        if (!ok) continue;
      }
      uint8_t* prow = sP[s] + r * 128;
#pragma unroll
      for (int cch = 0; cch < 16; ++cch) {
        const int q = cch >> 2, i0 = (cch & 3) * 8;
        uint4 u;
        u.x = pack_bf16(__uint_as_float(x[q][i0 + 0]), __uint_as_float(x[q][i0 + 1]));
        u.y = pack_bf16(__uint_as_float(x[q][i0 + 2]), __uint_as_float(x[q][i0 + 3]));
        u.z = pack_bf16(__uint_as_float(x[q][i0 + 4]), __uint_as_float(x[q][i0 + 5]));
        u.w = pack_bf16(__uint_as_float(x[q][i0 + 6]), __uint_as_float(x[q][i0 + 7]));
        const int half = cch >> 3, chunk = cch & 7;
        *reinterpret_cast<uint4*>(prow + half * kHalf + ((chunk ^ (r & 7)) << 4)) = u;
      }
      if (__any_sync(FULL, rescale)) {
        // O holds P_{<j} V_{<j} once P_{j-1} V_{j-1} has landed; rows that keep their
        // reference scale by 1 (exact), so the whole warp runs the TMEM round trip.
        const int jp = j - 1;
        ok = __all_sync(FULL, wait_bar(&bars.p_empty[jp & 1], (jp >> 1) & 1, abort));
        if (!ok) continue;
        tc05::fence_after_sync();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tc05::tmem_ld32(tO + lane_off + 32 * q, o);
          tc05::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tc05::tmem_st32(tO + lane_off + 32 * q, o);
        }
        tc05::tmem_wait_st();
      }
      tc05::fence_proxy_async_smem();
      tc05::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[s]);
    }
    // epilogue: O / l to global memory
    ok = __all_sync(FULL, ok && wait_bar(&bars.o_full, 0, abort));
    if (ok) {
      tc05::fence_after_sync();
      const float inv = 1.f / l;
      const int64_t qtok = int64_t(a.f_end - a.f_begin) * a.T;
      const int64_t row = int64_t(b) * qtok + qtok0 + r;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tc05::tmem_ld32(tO + lane_off + 32 * q, o);
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
  static unsigned configured = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 32) return cudaErrorInvalidDevice;
  if (!(configured & (1u << dev))) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured |= 1u << dev;
  }
  const int64_t grid = int64_t(a.fl.n_items) * (a.T / kBM) * a.H;
  prefill_tc_kernel<<<unsigned(grid), kThreads, kSmemBytes, s>>>(a, maps);
  return cudaGetLastError();
}

}  // namespace wam
