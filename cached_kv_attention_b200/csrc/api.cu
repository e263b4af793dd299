// C-ABI entry points: argument validation (before any CUDA call), construction of the
// per-launch work lists from the host padding mask and attention blocks, and dispatch to the
// tensor-core or CUDA-core kernels.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <functional>
#include <mutex>
#include <queue>
#include <string>
#include <vector>

#include <cudaTypedefs.h>

#include "launch.h"

// The device error word: kernels whose bounded waits give up write WAM_ERR_TIMEOUT here.
__device__ int g_wam_device_error = 0;

namespace {

thread_local std::string g_last_error;

// Address of the error word on the current device, looked up on every call: an address kept
// from an earlier call could belong to a context that a device reset has since replaced.
int* device_error_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_wam_device_error) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return static_cast<int*>(p);
}

wam_status fail(wam_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

wam_status ok() {
  g_last_error.clear();
  return WAM_OK;
}

wam_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(WAM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validated geometry with the derived per-episode valid-frame lists.
struct Geo {
  int B, H, D, T, F;
  std::vector<uint8_t> pad;     // [B*F]
  std::vector<int32_t> block;   // [F]
  std::vector<int> kf_end;      // [F]: first frame after the block of f
};

wam_status check_layout(const wam_video_layout* L, Geo& g) {
  if (!L) return fail(WAM_ERR_INVALID_ARGUMENT, "layout is NULL");
  if (L->B < 1 || L->H < 1 || L->T < 1 || L->F < 1)
    return fail(WAM_ERR_INVALID_ARGUMENT, "B, H, T, F must be >= 1 (got %d, %d, %d, %d)", L->B,
                L->H, L->T, L->F);
  if (L->D != 64 && L->D != 128)
    return fail(WAM_ERR_UNSUPPORTED, "head dim D must be 64 or 128 (got %d)", L->D);
  if (L->F > WAM_MAX_FRAMES)
    return fail(WAM_ERR_UNSUPPORTED, "F = %d exceeds WAM_MAX_FRAMES = %d", L->F, WAM_MAX_FRAMES);
  if (int64_t(L->B) * L->F > WAM_MAX_EPISODE_FRAMES)
    return fail(WAM_ERR_UNSUPPORTED, "B * F = %lld exceeds WAM_MAX_EPISODE_FRAMES = %d",
                (long long)L->B * L->F, WAM_MAX_EPISODE_FRAMES);
  if (int64_t(L->T) * L->F > (int64_t(1) << 24) || L->H > 4096)
    return fail(WAM_ERR_UNSUPPORTED, "F * T or H too large");
  g.B = L->B, g.H = L->H, g.D = L->D, g.T = L->T, g.F = L->F;
  g.pad.assign(size_t(g.B) * g.F, 0);
  if (L->frame_pad)
    for (size_t i = 0; i < g.pad.size(); ++i) {
      if (L->frame_pad[i] > 1)
        return fail(WAM_ERR_INVALID_ARGUMENT, "frame_pad[%zu] = %u is not 0 or 1", i,
                    unsigned(L->frame_pad[i]));
      g.pad[i] = L->frame_pad[i];
    }
  g.block.resize(g.F);
  for (int f = 0; f < g.F; ++f) {
    g.block[f] = L->frame_block ? L->frame_block[f] : f;
    if (f && g.block[f] < g.block[f - 1])
      return fail(WAM_ERR_INVALID_ARGUMENT, "frame_block must be nondecreasing (frame %d)", f);
  }
  g.kf_end.resize(g.F);
  for (int f = g.F - 1; f >= 0; --f)
    g.kf_end[f] = (f + 1 < g.F && g.block[f + 1] == g.block[f]) ? g.kf_end[f + 1] : f + 1;
  return WAM_OK;
}

wam_status check_dtype(wam_dtype dt, const char* name) {
  if (dt != WAM_F32 && dt != WAM_BF16)
    return fail(WAM_ERR_INVALID_ARGUMENT, "%s: unknown dtype %d", name, int(dt));
  return WAM_OK;
}

// Valid-frame lists of every episode.
void fill_vlists(const Geo& g, wam::FrameLists& fl) {
  for (int b = 0; b < g.B; ++b) {
    int n = 0;
    for (int f = 0; f < g.F; ++f)
      if (!g.pad[size_t(b) * g.F + f]) fl.vlist[b * g.F + n++] = uint16_t(f);
    fl.nvalid[b] = uint16_t(n);
  }
}

// Work items of a prefill call: every valid query frame in [f_begin, f_end), with the number
// of valid key frames it reads (those of blocks up to its own), longest first.
void fill_items(const Geo& g, int f_begin, int f_end, wam::FrameLists& fl) {
  std::vector<uint32_t> items;
  for (int b = 0; b < g.B; ++b)
    for (int f = f_begin; f < f_end; ++f) {
      if (g.pad[size_t(b) * g.F + f]) continue;
      int nk = 0;
      for (int u = 0; u < fl.nvalid[b]; ++u)
        if (fl.vlist[b * g.F + u] < g.kf_end[f]) ++nk;
      items.push_back(wam::pack_item(b, f, nk));
    }
  std::stable_sort(items.begin(), items.end(), [](uint32_t x, uint32_t y) {
    return wam::item_nk(x) > wam::item_nk(y);
  });
  fl.n_items = int32_t(items.size());
  std::copy(items.begin(), items.end(), fl.item);
}

// SM count of the current device (looked up once per device; concurrent first calls may both
// look it up and store the same value).
int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (!n) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

wam_status check_range(const Geo& g, int f_begin, int f_end) {
  if (f_begin < 0 || f_end > g.F || f_begin >= f_end)
    return fail(WAM_ERR_INVALID_ARGUMENT, "frame range [%d, %d) is not inside [0, %d)", f_begin,
                f_end, g.F);
  if (f_begin > 0 && g.block[f_begin - 1] == g.block[f_begin])
    return fail(WAM_ERR_INVALID_ARGUMENT, "f_begin = %d splits an attention block", f_begin);
  if (f_end < g.F && g.block[f_end - 1] == g.block[f_end])
    return fail(WAM_ERR_INVALID_ARGUMENT, "f_end = %d splits an attention block", f_end);
  return WAM_OK;
}

#define WAM_CHECK(expr)            \
  do {                             \
    wam_status st_ = (expr);       \
    if (st_ != WAM_OK) return st_; \
  } while (0)

#define WAM_NONNULL_ALIGNED(p)                                                             \
  do {                                                                                     \
    if (!(p)) return fail(WAM_ERR_INVALID_ARGUMENT, "%s is NULL", #p);                    \
    if (!aligned16(p)) return fail(WAM_ERR_INVALID_ARGUMENT, "%s is not 16-byte aligned", #p); \
  } while (0)

// Tensor-core eligibility of a bf16 video/action call.
bool tc_video_ok(const Geo& g, wam_dtype dt) { return dt == WAM_BF16 && g.D == 128 && g.T % 128 == 0; }

// Launch order of the tensor-core prefill's work items (one resident CTA per SM; the CTAs of
// an item are consecutive blocks).  The block scheduler hands blocks to SMs in index order
// as SMs free up, and a pass holds only a few CTAs per SM, so longest-first can end in a wave
// of short CTAs on a mostly idle GPU.  Candidates are longest-first and, for each class of
// equal key-frame count, that class moved right behind the longest class or to the end; each
// is scored by replaying that dispatch with a cost of (key tiles + a fixed 5-tile prologue
// and epilogue) per CTA.  The cheapest order is kept, longest-first on ties.  Results do not
// depend on the order: every CTA writes only its own rows.
void order_items_for_tc(const Geo& g, wam::FrameLists& fl, int sms) {
  constexpr int kOverheadTiles = 5;
  constexpr int64_t kMaxReplayBlocks = 60000;  // bound on host work per call
  const int n = fl.n_items;
  const int tpf = g.T / 128, QP = (g.T / 128 + 1) / 2;
  const int64_t per_item = int64_t(QP) * g.H;
  if (n < 2 || sms <= 0 || int64_t(n) * per_item <= sms) return;  // one wave: any order
  // Every layer of a pass has the same work list: the last answer is kept (per host thread)
  // and reused when the list, the SM count and the tile geometry all match.
  struct Memo {
    int sms = 0, tpf = 0;
    int64_t per_item = 0;
    std::vector<uint32_t> in, out;
  };
  static thread_local Memo memo;
  if (memo.sms == sms && memo.tpf == tpf && memo.per_item == per_item &&
      memo.in.size() == size_t(n) && std::equal(memo.in.begin(), memo.in.end(), fl.item)) {
    std::copy(memo.out.begin(), memo.out.end(), fl.item);
    return;
  }
  const std::vector<uint32_t> in(fl.item, fl.item + n);
  std::vector<int> nk;                          // classes, longest first (items are sorted)
  std::vector<std::vector<uint32_t>> members;
  for (int i = 0; i < n; ++i) {
    const int k = wam::item_nk(fl.item[i]);
    if (nk.empty() || nk.back() != k) nk.push_back(k), members.emplace_back();
    members.back().push_back(fl.item[i]);
  }
  const int C = int(nk.size());
  if (C < 2 || int64_t(2 * C - 1) * n * per_item > kMaxReplayBlocks) return;
  auto makespan = [&](const std::vector<int>& order) {
    std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> free_at;
    for (int i = 0; i < sms; ++i) free_at.push(0);
    int64_t end = 0;
    for (int c : order) {
      const int64_t cost = int64_t(nk[c]) * tpf + kOverheadTiles;
      for (int64_t m = int64_t(members[c].size()) * per_item; m > 0; --m) {
        const int64_t e = free_at.top() + cost;
        free_at.pop();
        free_at.push(e);
        end = std::max(end, e);
      }
    }
    return end;
  };
  std::vector<int> best(C);
  for (int c = 0; c < C; ++c) best[c] = c;
  int64_t best_t = makespan(best);
  const std::vector<int> lpt = best;
  for (int c = 1; c < C; ++c)
    for (int where : {1, C - 1}) {
      std::vector<int> o = lpt;
      o.erase(o.begin() + c);
      o.insert(o.begin() + where, c);
      const int64_t t = makespan(o);
      if (t < best_t) best_t = t, best = o;
    }
  int i = 0;
  for (int c : best)
    for (uint32_t it : members[c]) fl.item[i++] = it;
  memo.sms = sms, memo.tpf = tpf, memo.per_item = per_item;
  memo.in = in;
  memo.out.assign(fl.item, fl.item + n);
}
// Cross-frame pairing of a one-wave call.  When every CTA of a call is resident at once, its
// time is that of the longest CTA, and a CTA normally takes two query tiles of one frame: the
// frames with the most key frames set the time while the others finish early.  Paired, a CTA
// takes the same query tile of two frames of one episode, one with the most key frames and
// one with the fewest (items 2i and 2i + 1, fl.paired = 1): the second frame's keys are the
// first entries of the first one's, so the two tiles share every key tile up to the end of
// the shorter list, and only the rest runs for one tile.  Same number of CTAs; needs an even
// number of 128-row query tiles per frame and of items per episode, and unequal key counts.
void pair_items_for_tc(const Geo& g, wam::FrameLists& fl, int sms) {
  fl.paired = 0;
  const int QT = g.T / 128;
  if (QT % 2 || sms <= 0 || fl.n_items < 2) return;
  if (int64_t(fl.n_items) * (QT / 2) * g.H > sms) return;  // several waves: keep the order
  std::vector<std::vector<uint32_t>> per(g.B);
  for (int i = 0; i < fl.n_items; ++i) per[wam::item_b(fl.item[i])].push_back(fl.item[i]);
  bool unequal = false;
  for (auto& v : per) {
    if (v.size() % 2) return;
    std::stable_sort(v.begin(), v.end(),
                     [](uint32_t x, uint32_t y) { return wam::item_nk(x) > wam::item_nk(y); });
    if (!v.empty() && wam::item_nk(v.front()) != wam::item_nk(v.back())) unequal = true;
  }
  if (!unequal) return;
  int k = 0;
  for (auto& v : per)
    for (size_t i = 0; i < v.size() / 2; ++i) {
      fl.item[k++] = v[i];
      fl.item[k++] = v[v.size() - 1 - i];
    }
  fl.paired = 1;
}

bool tc_action_ok(const Geo& g, wam_dtype dt, int n_act) {
  return dt == WAM_BF16 && g.D == 128 && g.T % 64 == 0 && n_act <= 32;
}

}  // namespace

// ---------------------------------------------------------------------------------------
// tensor maps (driver entry point fetched through the runtime; no -lcuda)
// ---------------------------------------------------------------------------------------
namespace wam {
// Records a failure for wam_last_error() from entry points defined in other files.
wam_status record_error(wam_status st, const char* msg) { return fail(st, "%s", msg); }

bool make_tmap_bf16(CUtensorMap* map, const void* base, int B, int ntok, int H, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!encode) return false;
  const cuuint64_t dims[4] = {128, cuuint64_t(H), cuuint64_t(ntok), cuuint64_t(B)};
  const cuuint64_t strides[3] = {cuuint64_t(128) * 2, cuuint64_t(H) * 128 * 2,
                                 cuuint64_t(ntok) * H * 128 * 2};
  const cuuint32_t box[4] = {64, 1, cuuint32_t(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace wam

// ---------------------------------------------------------------------------------------
// entry points
// ---------------------------------------------------------------------------------------
extern "C" {

int32_t wam_version(void) { return 100; }

const char* wam_last_error(void) { return g_last_error.c_str(); }

wam_status wam_flow_schedule(int32_t n_steps, double sigma_end, double shift, double* sigmas) {
  if (n_steps < 1) return fail(WAM_ERR_INVALID_ARGUMENT, "n_steps must be >= 1");
  if (!sigmas) return fail(WAM_ERR_INVALID_ARGUMENT, "sigmas is NULL");
  if (!(shift > 0.0) || !std::isfinite(sigma_end) || sigma_end < 0.0 || sigma_end >= 1.0)
    return fail(WAM_ERR_INVALID_ARGUMENT, "need shift > 0 and 0 <= sigma_end < 1");
  for (int i = 0; i <= n_steps; ++i) {
    const double u = double(n_steps - i) / double(n_steps);
    const double phi = shift == 1.0 ? u : shift * u / (1.0 + (shift - 1.0) * u);
    sigmas[i] = sigma_end + (1.0 - sigma_end) * phi;
  }
  return ok();
}

wam_status wam_fuse_weights(int32_t n, const float* logits, float* weights) {
  if (n < 1 || n > WAM_MAX_FUSE_LAYERS)
    return fail(WAM_ERR_INVALID_ARGUMENT, "n must be in [1, %d]", WAM_MAX_FUSE_LAYERS);
  if (!logits || !weights) return fail(WAM_ERR_INVALID_ARGUMENT, "NULL pointer");
  double mx = -INFINITY;
  for (int i = 0; i < n; ++i) {
    if (std::isnan(logits[i]) || logits[i] == INFINITY)
      return fail(WAM_ERR_INVALID_ARGUMENT, "logit %d is not finite or -inf", i);
    mx = std::max(mx, double(logits[i]));
  }
  if (mx == -INFINITY) return fail(WAM_ERR_INVALID_ARGUMENT, "all logits are -inf");
  double e[WAM_MAX_FUSE_LAYERS], s = 0.0;
  for (int i = 0; i < n; ++i) s += (e[i] = std::exp(double(logits[i]) - mx));
  for (int i = 0; i < n; ++i) weights[i] = float(e[i] / s);
  return ok();
}

wam_status wam_flow_euler_step(int64_t n, float* x, const float* v, float dsigma,
                               wam_stream_t stream) {
  if (n < 0) return fail(WAM_ERR_INVALID_ARGUMENT, "n must be >= 0");
  if (n == 0) return ok();
  WAM_NONNULL_ALIGNED(x);
  WAM_NONNULL_ALIGNED(v);
  if (!std::isfinite(dsigma)) return fail(WAM_ERR_INVALID_ARGUMENT, "dsigma is not finite");
  return cuda_status(wam::launch_euler(n, x, v, dsigma, reinterpret_cast<cudaStream_t>(stream)),
                     "wam_flow_euler_step");
}

wam_status wam_copy_frames(const wam_video_layout* layout, wam_dtype dt, int32_t n,
                           const void* const* src, void* const* dst, int32_t f_src,
                           int32_t f_dst, int32_t n_frames, wam_stream_t stream) {
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  WAM_CHECK(check_dtype(dt, "dt"));
  if (n < 1 || n > WAM_MAX_COPY_TENSORS)
    return fail(WAM_ERR_INVALID_ARGUMENT, "n must be in [1, %d] (got %d)", WAM_MAX_COPY_TENSORS, n);
  if (!src || !dst) return fail(WAM_ERR_INVALID_ARGUMENT, "src or dst is NULL");
  if (n_frames < 0 || f_src < 0 || f_dst < 0 || f_src + n_frames > g.F || f_dst + n_frames > g.F)
    return fail(WAM_ERR_INVALID_ARGUMENT, "frames [%d, %d) -> [%d, %d) outside [0, %d)", f_src,
                f_src + n_frames, f_dst, f_dst + n_frames, g.F);
  const size_t es = dt == WAM_BF16 ? 2 : 4;
  const size_t frame_bytes = size_t(g.T) * g.H * g.D * es;
  const size_t tensor_bytes = size_t(g.B) * g.F * frame_bytes;
  static thread_local wam::CopyArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int j = 0; j < n; ++j) {
    if (!src[j] || !dst[j])
      return fail(WAM_ERR_INVALID_ARGUMENT, "src[%d] or dst[%d] is NULL", j, j);
    if (!aligned16(src[j]) || !aligned16(dst[j]))
      return fail(WAM_ERR_INVALID_ARGUMENT, "src[%d] or dst[%d] is not 16-byte aligned", j, j);
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(src[j]), d0 = reinterpret_cast<uintptr_t>(dst[j]);
    if (s0 < d0 + tensor_bytes && d0 < s0 + tensor_bytes)
      return fail(WAM_ERR_INVALID_ARGUMENT, "src[%d] and dst[%d] overlap", j, j);
    a.src[j] = src[j];
    a.dst[j] = dst[j];
  }
  if (n_frames == 0) return ok();
  a.n = n, a.B = g.B;
  a.ep_vec = int64_t(g.F) * frame_bytes / 16;
  a.src_vec = int64_t(f_src) * frame_bytes / 16;
  a.dst_vec = int64_t(f_dst) * frame_bytes / 16;
  a.n_vec = int64_t(n_frames) * frame_bytes / 16;
  return cuda_status(wam::launch_copy_frames(a, reinterpret_cast<cudaStream_t>(stream)),
                     "wam_copy_frames");
}

wam_status wam_video_prefill_kv(const wam_video_layout* layout, wam_dtype dt, int32_t f_begin,
                                int32_t f_end, const void* q, const void* k_new,
                                const void* v_new, void* k_cache, void* v_cache,
                                int32_t store_kv, void* o, wam_dtype o_dt,
                                const wam_fuse_epilogue* fuse, wam_stream_t stream) {
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  WAM_CHECK(check_dtype(dt, "dt"));
  WAM_CHECK(check_dtype(o_dt, "o_dt"));
  if (o_dt != WAM_F32 && o_dt != dt)
    return fail(WAM_ERR_UNSUPPORTED, "o_dt must be WAM_F32 or the input dtype");
  WAM_CHECK(check_range(g, f_begin, f_end));
  WAM_NONNULL_ALIGNED(q);
  WAM_NONNULL_ALIGNED(k_new);
  WAM_NONNULL_ALIGNED(v_new);
  WAM_NONNULL_ALIGNED(o);
  if (f_begin > 0 || store_kv) {
    WAM_NONNULL_ALIGNED(k_cache);
    WAM_NONNULL_ALIGNED(v_cache);
  }
  if (fuse) {
    if (!std::isfinite(fuse->weight))
      return fail(WAM_ERR_INVALID_ARGUMENT, "fuse->weight is not finite");
    if (!(fuse->first_in_interval && fuse->last_in_interval)) {
      WAM_NONNULL_ALIGNED(fuse->acc_k);
      WAM_NONNULL_ALIGNED(fuse->acc_v);
    }
    if (fuse->last_in_interval) {
      WAM_NONNULL_ALIGNED(fuse->fused_k);
      WAM_NONNULL_ALIGNED(fuse->fused_v);
    }
  }
  static thread_local wam::PrefillArgs a;  // large; built on the host per call
  std::memset(&a, 0, sizeof(a));
  a.q = q, a.k_new = k_new, a.v_new = v_new, a.k_cache = k_cache, a.v_cache = v_cache;
  a.k_store = store_kv ? k_cache : nullptr;
  a.v_store = store_kv ? v_cache : nullptr;
  a.o = o;
  if (fuse) {
    a.fuse_on = 1, a.fuse_first = fuse->first_in_interval ? 1 : 0;
    a.fuse_last = fuse->last_in_interval ? 1 : 0, a.fuse_w = fuse->weight;
    a.acc_k = fuse->acc_k, a.acc_v = fuse->acc_v, a.fused_k = fuse->fused_k, a.fused_v = fuse->fused_v;
  }
  a.B = g.B, a.H = g.H, a.T = g.T, a.F = g.F, a.f_begin = f_begin, a.f_end = f_end;
  a.o_f32 = o_dt == WAM_F32;
  a.scale_log2 = float(wam::kLog2e / std::sqrt(double(g.D)));
  a.err = device_error_word();
  fill_vlists(g, a.fl);
  fill_items(g, f_begin, f_end, a.fl);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool bf16 = dt == WAM_BF16;
  if (tc_video_ok(g, dt)) {
    order_items_for_tc(g, a.fl, sm_count());
    pair_items_for_tc(g, a.fl, sm_count());
    cudaError_t e = wam::launch_prefill_tc(a, s);
    if (e != cudaErrorNotSupported) return cuda_status(e, "wam_video_prefill_kv (tensor cores)");
  }
  cudaError_t e = wam::launch_prefill_simt(a, g.D, bf16, s);
  if (e == cudaSuccess) e = wam::launch_store_fuse(a, g.D, bf16, s);
  return cuda_status(e, "wam_video_prefill_kv");
}

wam_status wam_fuse_interval_kv(const wam_video_layout* layout, wam_dtype dt, int32_t n_layers,
                                const void* const* k_layers, const void* const* v_layers,
                                const float* weights, int32_t f_begin, int32_t f_end,
                                void* fused_k, void* fused_v, wam_stream_t stream) {
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  WAM_CHECK(check_dtype(dt, "dt"));
  if (n_layers < 1 || n_layers > WAM_MAX_FUSE_LAYERS)
    return fail(WAM_ERR_INVALID_ARGUMENT, "n_layers must be in [1, %d]", WAM_MAX_FUSE_LAYERS);
  if (!k_layers || !v_layers || !weights)
    return fail(WAM_ERR_INVALID_ARGUMENT, "k_layers, v_layers and weights must not be NULL");
  if (f_begin < 0 || f_end > g.F || f_begin >= f_end)
    return fail(WAM_ERR_INVALID_ARGUMENT, "frame range [%d, %d) is not inside [0, %d)", f_begin,
                f_end, g.F);
  WAM_NONNULL_ALIGNED(fused_k);
  WAM_NONNULL_ALIGNED(fused_v);
  static thread_local wam::FuseArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int l = 0; l < n_layers; ++l) {
    if (!k_layers[l] || !v_layers[l] || !aligned16(k_layers[l]) || !aligned16(v_layers[l]))
      return fail(WAM_ERR_INVALID_ARGUMENT, "layer %d pointer is NULL or not 16-byte aligned", l);
    if (!std::isfinite(weights[l]))
      return fail(WAM_ERR_INVALID_ARGUMENT, "weight %d is not finite", l);
    a.k[l] = k_layers[l], a.v[l] = v_layers[l], a.w[l] = weights[l];
  }
  a.n_layers = n_layers, a.fk = fused_k, a.fv = fused_v, a.F = g.F;
  a.frame_elems = int64_t(g.T) * g.H * g.D;
  std::vector<uint32_t> items;
  for (int b = 0; b < g.B; ++b)
    for (int f = f_begin; f < f_end; ++f)
      if (!g.pad[size_t(b) * g.F + f]) items.push_back(wam::pack_item(b, f, 0));
  a.fl.n_items = int32_t(items.size());
  std::copy(items.begin(), items.end(), a.fl.item);
  return cuda_status(wam::launch_fuse(a, g.D, dt == WAM_BF16, reinterpret_cast<cudaStream_t>(stream)),
                     "wam_fuse_interval_kv");
}

// Geometry of the persistent tensor-core action read: tiles G, CTAs P, partial slots.
static wam_status action_plan(wam::ActionArgs& a, size_t* bytes) {
  const int sms = sm_count();
  if (sms <= 0) return fail(WAM_ERR_CUDA, "wam_action_attn: no CUDA device");
  if (int64_t(a.B) * a.H * int64_t(sizeof(int)) > int64_t(wam::kTicketBytes))
    return fail(WAM_ERR_UNSUPPORTED, "wam_action_attn: B * H exceeds %d", int(wam::kTicketBytes / sizeof(int)));
  if (a.T % 128 == 0) {
    wam::action_aligned_plan(a, sms);  // the 128-key tensor-core reads
  } else {
    a.G = wam::action_tc_total_tiles(a);  // the 64-key mma.sync read: a flat split
    a.P = a.G < sms ? a.G : sms;
    a.max_parts = wam::action_tc_max_parts(a, a.P, a.G);
  }
  *bytes = wam::action_tc_workspace_bytes(a.B * a.H, a.max_parts);
  return WAM_OK;
}

wam_status wam_action_attn_workspace_size(const wam_video_layout* layout, wam_dtype dt,
                                          int32_t n_act, int32_t with_video, size_t* bytes) {
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  WAM_CHECK(check_dtype(dt, "dt"));
  if (!bytes) return fail(WAM_ERR_INVALID_ARGUMENT, "bytes is NULL");
  if (n_act < 1 || n_act > 128)
    return fail(WAM_ERR_INVALID_ARGUMENT, "n_act must be in [1, 128] (got %d)", n_act);
  *bytes = 0;
  if (!tc_action_ok(g, dt, n_act)) return ok();
  static thread_local wam::ActionArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = g.B, a.H = g.H, a.T = g.T, a.F = g.F, a.n_act = n_act, a.with_video = with_video ? 1 : 0;
  fill_vlists(g, a.fl);
  WAM_CHECK(action_plan(a, bytes));
  return ok();
}

wam_status wam_action_attn(const wam_video_layout* layout, wam_dtype dt, const void* fused_k,
                           const void* fused_v, int32_t n_act, const void* qa, const void* ka,
                           const void* va, void* o, wam_dtype o_dt, void* workspace,
                           size_t ws_bytes, wam_stream_t stream) {
  return wam_action_attn_ex(layout, dt, fused_k, fused_v, n_act, qa, ka, va, o, o_dt, workspace,
                            ws_bytes, 0u, stream);
}

wam_status wam_action_attn_ex(const wam_video_layout* layout, wam_dtype dt, const void* fused_k,
                              const void* fused_v, int32_t n_act, const void* qa, const void* ka,
                              const void* va, void* o, wam_dtype o_dt, void* workspace,
                              size_t ws_bytes, uint32_t flags, wam_stream_t stream) {
  if (flags & ~uint32_t(WAM_ACTION_FUSED_READY))
    return fail(WAM_ERR_INVALID_ARGUMENT, "unknown flags 0x%x", unsigned(flags));
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  WAM_CHECK(check_dtype(dt, "dt"));
  WAM_CHECK(check_dtype(o_dt, "o_dt"));
  if (o_dt != WAM_F32 && o_dt != dt)
    return fail(WAM_ERR_UNSUPPORTED, "o_dt must be WAM_F32 or the input dtype");
  if (n_act < 1 || n_act > 128)
    return fail(WAM_ERR_INVALID_ARGUMENT, "n_act must be in [1, 128] (got %d)", n_act);
  if ((fused_k == nullptr) != (fused_v == nullptr))
    return fail(WAM_ERR_INVALID_ARGUMENT, "fused_k and fused_v must both be set or both NULL");
  if (fused_k) {
    WAM_NONNULL_ALIGNED(fused_k);
    WAM_NONNULL_ALIGNED(fused_v);
  }
  WAM_NONNULL_ALIGNED(qa);
  WAM_NONNULL_ALIGNED(ka);
  WAM_NONNULL_ALIGNED(va);
  WAM_NONNULL_ALIGNED(o);
  static thread_local wam::ActionArgs a;
  std::memset(&a, 0, sizeof(a));
  a.fk = fused_k, a.fv = fused_v, a.qa = qa, a.ka = ka, a.va = va, a.o = o;
  a.B = g.B, a.H = g.H, a.T = g.T, a.F = g.F, a.n_act = n_act;
  a.o_f32 = o_dt == WAM_F32;
  a.with_video = fused_k != nullptr;
  a.fused_ready = (flags & WAM_ACTION_FUSED_READY) ? 1 : 0;
  a.scale_log2 = float(wam::kLog2e / std::sqrt(double(g.D)));
  a.err = device_error_word();
  fill_vlists(g, a.fl);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (tc_action_ok(g, dt, n_act)) {
    size_t need = 0;
    WAM_CHECK(action_plan(a, &need));
    if (need) {
      if (!workspace || ws_bytes < need)
        return fail(WAM_ERR_WORKSPACE, "wam_action_attn: workspace of %zu bytes needed (got %zu)",
                    need, workspace ? ws_bytes : size_t(0));
      if (!aligned16(workspace))
        return fail(WAM_ERR_INVALID_ARGUMENT, "workspace is not 16-byte aligned");
      a.ws_count = static_cast<int*>(workspace);
      a.ws_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + wam::kTicketBytes);
    }
    cudaError_t e = wam::launch_action_tc(a, s);
    if (e != cudaErrorNotSupported) return cuda_status(e, "wam_action_attn (tensor cores)");
  }
  return cuda_status(wam::launch_action_simt(a, g.D, dt == WAM_BF16, s), "wam_action_attn");
}

wam_status wam_action_attn_nvfp4(const wam_video_layout* layout, const void* k_codes,
                                 const void* k_scales, const float* k_sg, const void* v_codes,
                                 const void* v_scales, const float* v_sg, int32_t n_act,
                                 const void* qa, const void* ka, const void* va, void* o,
                                 wam_dtype o_dt, void* workspace, size_t ws_bytes,
                                 uint32_t flags, wam_stream_t stream) {
  if (flags & ~uint32_t(WAM_ACTION_FUSED_READY))
    return fail(WAM_ERR_INVALID_ARGUMENT, "unknown flags 0x%x", unsigned(flags));
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  WAM_CHECK(check_dtype(o_dt, "o_dt"));
  if (g.D != 128 || g.T % 128 != 0)
    return fail(WAM_ERR_UNSUPPORTED, "wam_action_attn_nvfp4 needs D = 128 and T %% 128 == 0 (got D = %d, T = %d)",
                g.D, g.T);
  if (n_act < 1 || n_act > 32)
    return fail(WAM_ERR_UNSUPPORTED, "wam_action_attn_nvfp4 needs 1 <= n_act <= 32 (got %d)", n_act);
  WAM_NONNULL_ALIGNED(k_codes);
  WAM_NONNULL_ALIGNED(k_scales);
  WAM_NONNULL_ALIGNED(v_codes);
  WAM_NONNULL_ALIGNED(v_scales);
  if (!k_sg || !v_sg) return fail(WAM_ERR_INVALID_ARGUMENT, "k_sg or v_sg is NULL");
  if ((reinterpret_cast<uintptr_t>(k_sg) & 3u) || (reinterpret_cast<uintptr_t>(v_sg) & 3u))
    return fail(WAM_ERR_INVALID_ARGUMENT, "k_sg or v_sg is not 4-byte aligned");
  WAM_NONNULL_ALIGNED(qa);
  WAM_NONNULL_ALIGNED(ka);
  WAM_NONNULL_ALIGNED(va);
  WAM_NONNULL_ALIGNED(o);
  static thread_local wam::ActionArgs a;
  std::memset(&a, 0, sizeof(a));
  a.qa = qa, a.ka = ka, a.va = va, a.o = o;
  a.k_codes = static_cast<const uint8_t*>(k_codes), a.k_scales = static_cast<const uint8_t*>(k_scales);
  a.v_codes = static_cast<const uint8_t*>(v_codes), a.v_scales = static_cast<const uint8_t*>(v_scales);
  a.k_sg = k_sg, a.v_sg = v_sg;
  a.B = g.B, a.H = g.H, a.T = g.T, a.F = g.F, a.n_act = n_act;
  a.o_f32 = o_dt == WAM_F32;
  a.with_video = 1;
  a.fused_ready = (flags & WAM_ACTION_FUSED_READY) ? 1 : 0;
  a.scale_log2 = float(wam::kLog2e / std::sqrt(double(g.D)));
  a.err = device_error_word();
  fill_vlists(g, a.fl);
  size_t need = 0;
  WAM_CHECK(action_plan(a, &need));
  if (need) {
    if (!workspace || ws_bytes < need)
      return fail(WAM_ERR_WORKSPACE, "wam_action_attn_nvfp4: workspace of %zu bytes needed (got %zu)", need,
                  workspace ? ws_bytes : size_t(0));
    if (!aligned16(workspace)) return fail(WAM_ERR_INVALID_ARGUMENT, "workspace is not 16-byte aligned");
    a.ws_count = static_cast<int*>(workspace);
    a.ws_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + wam::kTicketBytes);
  }
  return cuda_status(wam::launch_action_nvfp4(a, reinterpret_cast<cudaStream_t>(stream)),
                     "wam_action_attn_nvfp4");
}

wam_status wam_debug_video_mask(const wam_video_layout* layout, int32_t f_begin, int32_t f_end,
                                uint8_t* mask, wam_stream_t stream) {
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  WAM_CHECK(check_range(g, f_begin, f_end));
  if (!mask) return fail(WAM_ERR_INVALID_ARGUMENT, "mask is NULL");
  static thread_local wam::PrefillArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = g.B, a.H = g.H, a.T = g.T, a.F = g.F, a.f_begin = f_begin, a.f_end = f_end;
  fill_vlists(g, a.fl);
  fill_items(g, f_begin, f_end, a.fl);
  return cuda_status(wam::launch_debug_mask(a, mask, reinterpret_cast<cudaStream_t>(stream)),
                     "wam_debug_video_mask");
}

wam_status wam_debug_action_plan(const wam_video_layout* layout, int32_t n_sms, int32_t* kparts,
                                 int32_t* n_ctas, int32_t* max_parts) {
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  if (!kparts || !n_ctas || !max_parts)
    return fail(WAM_ERR_INVALID_ARGUMENT, "an output pointer is NULL");
  if (n_sms < 1) return fail(WAM_ERR_INVALID_ARGUMENT, "n_sms must be >= 1");
  if (g.T % 128 != 0)
    return fail(WAM_ERR_INVALID_ARGUMENT, "T = %d is not a multiple of 128", g.T);
  static thread_local wam::ActionArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = g.B, a.H = g.H, a.T = g.T, a.F = g.F, a.with_video = 1;
  fill_vlists(g, a.fl);
  *n_ctas = wam::action_aligned_plan(a, n_sms);
  *max_parts = a.max_parts;
  for (int b = 0; b < g.B; ++b) kparts[b] = a.kparts[b];
  return ok();
}

wam_status wam_debug_prefill_order(const wam_video_layout* layout, int32_t f_begin, int32_t f_end,
                                   int32_t n_sms, int32_t* episode, int32_t* frame,
                                   int32_t* n_key_frames, int32_t* n_items, int32_t* paired) {
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  WAM_CHECK(check_range(g, f_begin, f_end));
  if (!episode || !frame || !n_key_frames || !n_items)
    return fail(WAM_ERR_INVALID_ARGUMENT, "an output pointer is NULL");
  if (g.T % 128 != 0)
    return fail(WAM_ERR_INVALID_ARGUMENT, "T = %d is not a multiple of 128", g.T);
  static thread_local wam::PrefillArgs a;
  std::memset(&a, 0, sizeof(a));
  fill_vlists(g, a.fl);
  fill_items(g, f_begin, f_end, a.fl);
  order_items_for_tc(g, a.fl, n_sms);
  pair_items_for_tc(g, a.fl, n_sms);
  if (paired) *paired = a.fl.paired;
  for (int i = 0; i < a.fl.n_items; ++i) {
    episode[i] = wam::item_b(a.fl.item[i]);
    frame[i] = wam::item_f(a.fl.item[i]);
    n_key_frames[i] = wam::item_nk(a.fl.item[i]);
  }
  *n_items = a.fl.n_items;
  return WAM_OK;
}

wam_status wam_nvfp4_workspace_size(int32_t n, size_t* bytes) {
  if (n < 1 || n > WAM_MAX_NVFP4_TENSORS)
    return fail(WAM_ERR_INVALID_ARGUMENT, "n must be in [1, %d] (got %d)", WAM_MAX_NVFP4_TENSORS, n);
  if (!bytes) return fail(WAM_ERR_INVALID_ARGUMENT, "bytes is NULL");
  *bytes = size_t(n) * wam::kNvfp4MaxSlices * sizeof(float);
  return ok();
}

wam_status wam_fused_to_nvfp4(const wam_video_layout* layout, int32_t n, const void* const* fused,
                              void* const* codes, void* const* scales, float* s_g,
                              void* workspace, size_t ws_bytes, wam_stream_t stream) {
  Geo g;
  WAM_CHECK(check_layout(layout, g));
  if (n < 1 || n > WAM_MAX_NVFP4_TENSORS)
    return fail(WAM_ERR_INVALID_ARGUMENT, "n must be in [1, %d] (got %d)", WAM_MAX_NVFP4_TENSORS, n);
  if (!fused || !codes || !scales) return fail(WAM_ERR_INVALID_ARGUMENT, "fused, codes or scales is NULL");
  WAM_NONNULL_ALIGNED(s_g);
  size_t need = 0;
  WAM_CHECK(wam_nvfp4_workspace_size(n, &need));
  if (!workspace || ws_bytes < need)
    return fail(WAM_ERR_WORKSPACE, "wam_fused_to_nvfp4: workspace of %zu bytes needed (got %zu)", need,
                workspace ? ws_bytes : size_t(0));
  if (!aligned16(workspace)) return fail(WAM_ERR_INVALID_ARGUMENT, "workspace is not 16-byte aligned");
  static thread_local wam::Nvfp4Args a;
  std::memset(&a, 0, sizeof(a));
  for (int j = 0; j < n; ++j) {
    if (!fused[j] || !codes[j] || !scales[j])
      return fail(WAM_ERR_INVALID_ARGUMENT, "fused[%d], codes[%d] or scales[%d] is NULL", j, j, j);
    if (!aligned16(fused[j]) || !aligned16(codes[j]) || !aligned16(scales[j]))
      return fail(WAM_ERR_INVALID_ARGUMENT, "fused[%d], codes[%d] or scales[%d] is not 16-byte aligned", j, j, j);
    a.src[j] = fused[j], a.codes[j] = codes[j], a.scales[j] = scales[j];
  }
  a.s_g = s_g;
  a.ws = static_cast<float*>(workspace);
  a.n = n, a.B = g.B, a.H = g.H, a.D = g.D, a.T = g.T, a.F = g.F;
  a.frame_elems = int64_t(g.T) * g.H * g.D;
  std::vector<uint32_t> items;
  for (int b = 0; b < g.B; ++b)
    for (int f = 0; f < g.F; ++f)
      if (!g.pad[size_t(b) * g.F + f]) items.push_back(wam::pack_item(b, f, 0));
  a.fl.n_items = int32_t(items.size());
  std::copy(items.begin(), items.end(), a.fl.item);
  return cuda_status(wam::launch_nvfp4_encode(a, reinterpret_cast<cudaStream_t>(stream)),
                     "wam_fused_to_nvfp4");
}

wam_status wam_debug_wait_timeout(int32_t polls, wam_stream_t stream) {
  if (polls < 1 || uint32_t(polls) > wam::kWaitSpinLimit)
    return fail(WAM_ERR_INVALID_ARGUMENT, "polls must be in [1, %u] (got %d)",
                unsigned(wam::kWaitSpinLimit), polls);
  int* err = device_error_word();
  if (!err) return fail(WAM_ERR_CUDA, "wam_debug_wait_timeout: no device error word");
  return cuda_status(wam::launch_wait_timeout(uint32_t(polls), err,
                                              reinterpret_cast<cudaStream_t>(stream)),
                     "wam_debug_wait_timeout");
}

wam_status wam_device_error(int32_t clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e, "wam_device_error: synchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_wam_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_status(e, "wam_device_error: read");
  if (clear && v) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_wam_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_status(e, "wam_device_error: clear");
  }
  if (v) return fail(wam_status(v), "a kernel's bounded wait gave up (device error word = %d)", v);
  return ok();
}

}  // extern "C"
