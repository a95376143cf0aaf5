// C-ABI entry points of libsplitkv_attn: argument validation, per-batch
// tensor-map encoding (extents clipped to the valid keys / query rows of each
// batch row), launch on the caller's stream.  See include/splitkv_attn.h for
// the contract of every function.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>
#include <cstddef>

#include "../../include/splitkv_attn.h"
#include "attn_common.cuh"
#include "attn_fwd_persistent.cuh"
#include "qk_norm_rope.cuh"
#include "shard_copy.cuh"

namespace {

constexpr int32_t kAbiVersion = 2;

// ---------------------------------------------------------------- errors
thread_local std::string g_last_error;

sk_status_t fail(sk_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

sk_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(SK_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ---------------------------------------------------------------- device state
// The status word is a module global: one per device, no allocation.
__device__ int32_t g_device_status = 0;

uint64_t g_wait_limit_ns = 2000ull * 1000ull * 1000ull;
int32_t g_test_stall = 0;
std::mutex g_mu;

struct DeviceInfo {
  bool checked = false;
  bool sm100 = false;
  int sm_count = 0;
  int32_t* status = nullptr;
  bool attn_attr_set[8] = {};  // per kernel instance: cudaFuncSetAttribute done
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];

sk_status_t device_setup(int* dev_out, DeviceInfo** info_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SK_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    d.sm100 = (major == 10 && minor == 0);
    e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_device_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    d.status = static_cast<int32_t*>(ptr);
    d.checked = true;
  }
  if (!d.sm100) return fail(SK_ERR_UNSUPPORTED, "device %d is not sm_100 (B200)", dev);
  *dev_out = dev;
  *info_out = &d;
  return SK_OK;
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over (d, head, seq) of one batch row: box = 64 d x 1 head x 128 rows,
// 128-byte swizzle.  `rows` is the clipped sequence extent (>= 1).
//
// An encoded map is a pure function of its inputs (address, extents,
// strides; type, box and swizzle are fixed here), so encoded maps are kept in
// a small per-thread cache keyed on exactly those inputs: a caller that
// passes the same buffers again (the caching allocator hands the same
// addresses back every step) skips the driver's encoder.
struct MapKey {
  const void* base;
  int64_t stride_s, stride_h, rows;
  int32_t heads, D;
  bool operator==(const MapKey& o) const {
    return base == o.base && stride_s == o.stride_s && stride_h == o.stride_h && rows == o.rows &&
           heads == o.heads && D == o.D;
  }
};

struct MapCache {
  static constexpr int kWays = 64;
  MapKey key[kWays];
  CUtensorMap map[kWays];
  uint32_t stamp[kWays] = {};
  uint32_t clock = 0;
  bool valid[kWays] = {};
};
thread_local MapCache g_map_cache;

sk_status_t encode_map(CUtensorMap* m, const void* base, int64_t stride_s, int64_t stride_h,
                       int heads, int64_t rows, int D) {
  const MapKey k{base, stride_s, stride_h, rows, heads, D};
  MapCache& c = g_map_cache;
  int victim = -1;  // an empty slot if there is one, else the least recently used
  for (int i = 0; i < MapCache::kWays; ++i) {
    if (!c.valid[i]) {
      if (victim < 0 || c.valid[victim]) victim = i;
      continue;
    }
    if (c.key[i] == k) {
      c.stamp[i] = ++c.clock;
      *m = c.map[i];
      return SK_OK;
    }
    if (victim < 0 || (c.valid[victim] && c.stamp[i] < c.stamp[victim])) victim = i;
  }
  auto enc = get_encode_fn();
  if (!enc) return fail(SK_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(stride_h) * 2u, static_cast<cuuint64_t>(stride_s) * 2u};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(skattn::kBlockM)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SK_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  c.key[victim] = k;
  c.map[victim] = *m;
  c.valid[victim] = true;
  c.stamp[victim] = ++c.clock;
  return SK_OK;
}

// ---------------------------------------------------------------- validation helpers
struct Span {
  uintptr_t lo = 0, hi = 0;  // [lo, hi) bytes; empty when lo == hi
};

bool span_of(const sk_tensor_t& t, int B, int H, int D, Span* sp) {
  if (t.len_s == 0 || B == 0) {
    *sp = Span{};
    return true;
  }
  const uintptr_t base = reinterpret_cast<uintptr_t>(t.ptr);
  int64_t lo = 0, hi = 0;  // element offsets
  const int64_t ext[3] = {B - 1, static_cast<int64_t>(t.len_s) - 1, H - 1};
  const int64_t str[3] = {t.stride_b, t.stride_s, t.stride_h};
  for (int i = 0; i < 3; ++i) {
    const int64_t v = ext[i] * str[i];
    if (v < 0) lo += v; else hi += v;
  }
  hi += D;
  sp->lo = base + static_cast<uintptr_t>(lo * 2);
  sp->hi = base + static_cast<uintptr_t>(hi * 2);
  return true;
}

bool overlaps(const Span& a, const Span& b) {
  if (a.lo == a.hi || b.lo == b.hi) return false;
  return a.lo < b.hi && b.lo < a.hi;
}

// True when distinct (b, s, h, d) indices map to distinct elements (sufficient test:
// sorted by stride, every stride covers the span of all smaller dimensions).
bool no_self_overlap(const sk_tensor_t& t, int B, int H, int D) {
  struct Dim { int64_t n, st; } dims[3] = {{B, t.stride_b}, {t.len_s, t.stride_s}, {H, t.stride_h}};
  std::sort(dims, dims + 3, [](const Dim& a, const Dim& b) { return a.st < b.st; });
  int64_t span = D;  // d is contiguous
  for (auto& d : dims) {
    if (d.n <= 1) continue;
    if (d.st < span) return false;
    span = d.st * (d.n - 1) + span;
  }
  return true;
}

sk_status_t check_tensor(const char* name, const sk_tensor_t* t, int B, int H, int D) {
  if (!t) return fail(SK_ERR_INVALID_ARG, "%s: NULL descriptor", name);
  if (t->len_s < 0) return fail(SK_ERR_INVALID_ARG, "%s: negative len_s", name);
  if (t->len_s == 0 || B == 0) return SK_OK;
  if (!t->ptr) return fail(SK_ERR_INVALID_ARG, "%s: NULL ptr with len_s > 0", name);
  if (reinterpret_cast<uintptr_t>(t->ptr) % 16 != 0)
    return fail(SK_ERR_INVALID_ARG, "%s: ptr not 16-byte aligned", name);
  const int64_t st[3] = {t->stride_b, t->stride_s, t->stride_h};
  const char* nm[3] = {"stride_b", "stride_s", "stride_h"};
  for (int i = 0; i < 3; ++i) {
    if (st[i] % 8 != 0) return fail(SK_ERR_INVALID_ARG, "%s: %s=%lld not a multiple of 8 elements", name, nm[i], (long long)st[i]);
    if (st[i] < 0) return fail(SK_ERR_INVALID_ARG, "%s: %s negative", name, nm[i]);
    if (st[i] * 2 >= (int64_t(1) << 40)) return fail(SK_ERR_INVALID_ARG, "%s: %s too large", name, nm[i]);
  }
  if (H > 1 && t->stride_h == 0) return fail(SK_ERR_INVALID_ARG, "%s: stride_h is 0", name);
  if (t->len_s > 1 && t->stride_s == 0) return fail(SK_ERR_INVALID_ARG, "%s: stride_s is 0", name);
  return SK_OK;
}

template <int D>
sk_status_t set_smem(const void* kernel, int slot, uint32_t bytes, DeviceInfo* dev, int launch_regs = 0) {
  if (!dev->attn_attr_set[slot]) {
    if (launch_regs > 0) {
      // The kernel moves registers between its warpgroups (setmaxnreg); that
      // split adds up only if it is launched with exactly this many.
      cudaFuncAttributes a;
      cudaError_t e = cudaFuncGetAttributes(&a, kernel);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
      if (a.numRegs != launch_regs)
        return fail(SK_ERR_UNSUPPORTED, "attention kernel built with %d registers per thread, %d expected",
                    a.numRegs, launch_regs);
    }
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    dev->attn_attr_set[slot] = true;
  }
  return SK_OK;
}

template <int D>
sk_status_t launch_attn(skattn::AttnParams& prm, int n_qtiles, int H, int nb, cudaStream_t stream,
                        DeviceInfo* dev) {
  using L = skattn::PSmemLayout<D>;
  using P = skattn::AttnParams;
  const bool scatter = prm.out_chunk > 0;  // separate instance: the plain kernel's code is untouched
  const int slot = (D == 64 ? 0 : 1) + (scatter ? 2 : 0);
  auto kernel = scatter ? skattn::attn_fwd_persistent_kernel<D, true, P> : skattn::attn_fwd_persistent_kernel<D, false, P>;
  sk_status_t st;
  if ((st = set_smem<D>(reinterpret_cast<const void*>(kernel), slot, L::kAlloc, dev, skattn::kLaunchRegs)) != SK_OK)
    return st;
  prm.n_heads = H;
  prm.n_pairs = n_qtiles;
  const int64_t units = static_cast<int64_t>(nb) * H * n_qtiles;
  if (units > INT32_MAX) return fail(SK_ERR_UNSUPPORTED, "too many work units (%lld)", (long long)units);
  prm.n_units = static_cast<int32_t>(units);
  const int grid = static_cast<int>(std::min<int64_t>(units, dev->sm_count));
  kernel<<<grid, skattn::kPThreads, L::kAlloc, stream>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  return SK_OK;
}

// Output rows scattered over destination buffers (the output all-to-all of
// the Ulysses form): row s -> dst[s / layout.len_s], row s % layout.len_s,
// head head_offset + h; every destination has layout's strides.
struct ScatterOut {
  void* const* dst;
  int32_t n;
  const sk_tensor_t* layout;
  int32_t head_offset;
};

sk_status_t attn_impl(const sk_tensor_t* q, const sk_tensor_t* kp, const sk_tensor_t* vp,
                      const sk_tensor_t* ks, const sk_tensor_t* vs, const int32_t* real_len,
                      int32_t Hq, int32_t Hkv, float scale, const sk_tensor_t* out, int32_t B,
                      int32_t D, const int32_t* q_valid_in, void* stream_v,
                      const ScatterOut* scatter = nullptr) {
  if (B < 0) return fail(SK_ERR_INVALID_ARG, "batch < 0");
  if (Hq <= 0 || Hkv <= 0) return fail(SK_ERR_INVALID_ARG, "head counts must be positive");
  if (Hq % Hkv != 0) return fail(SK_ERR_INVALID_ARG, "num_q_heads %% num_kv_heads != 0");
  if (Hq > 65535) return fail(SK_ERR_UNSUPPORTED, "num_q_heads > 65535");
  if (D != 64 && D != 128) return fail(SK_ERR_UNSUPPORTED, "head_dim %d not in {64, 128}", D);
  if (!(std::isfinite(scale) && scale >= 0.f)) return fail(SK_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  sk_status_t st;
  if ((st = check_tensor("q", q, B, Hq, D)) != SK_OK) return st;
  if ((st = check_tensor("k_prefix", kp, B, Hkv, D)) != SK_OK) return st;
  if ((st = check_tensor("v_prefix", vp, B, Hkv, D)) != SK_OK) return st;
  if ((st = check_tensor("k_suffix", ks, B, Hkv, D)) != SK_OK) return st;
  if ((st = check_tensor("v_suffix", vs, B, Hkv, D)) != SK_OK) return st;
  const int32_t Sq = q->len_s;
  sk_tensor_t scatter_view;  // one destination as a tensor, for the stride checks
  if (scatter) {
    if (scatter->n < 1 || scatter->n > skattn::kMaxOutDst)
      return fail(SK_ERR_INVALID_ARG, "num_dst=%d outside [1, %d]", scatter->n, skattn::kMaxOutDst);
    if (!scatter->dst || !scatter->layout) return fail(SK_ERR_INVALID_ARG, "NULL destination array or layout");
    if (scatter->head_offset < 0) return fail(SK_ERR_INVALID_ARG, "head_offset < 0");
    const int32_t chunk = scatter->layout->len_s;
    if (chunk <= 0 || static_cast<int64_t>(chunk) * scatter->n != Sq)
      return fail(SK_ERR_INVALID_ARG, "num_dst (%d) x dst rows (%d) != q.len_s (%d)", scatter->n, chunk, Sq);
    for (int r = 0; r < scatter->n; ++r) {
      if (!scatter->dst[r]) return fail(SK_ERR_INVALID_ARG, "destination %d is NULL", r);
      if (reinterpret_cast<uintptr_t>(scatter->dst[r]) % 16)
        return fail(SK_ERR_INVALID_ARG, "destination %d not 16-byte aligned", r);
    }
    scatter_view = *scatter->layout;
    scatter_view.ptr = scatter->dst[0];
    if ((st = check_tensor("dst", &scatter_view, B, scatter->head_offset + Hq, D)) != SK_OK) return st;
    if (!no_self_overlap(scatter_view, B, scatter->head_offset + Hq, D))
      return fail(SK_ERR_INVALID_ARG, "destination layout overlaps itself");
    out = &scatter_view;
  } else {
    if ((st = check_tensor("out", out, B, Hq, D)) != SK_OK) return st;
    if (out->len_s != Sq) return fail(SK_ERR_INVALID_ARG, "out.len_s (%d) != q.len_s (%d)", out->len_s, Sq);
  }
  if (kp->len_s != vp->len_s) return fail(SK_ERR_INVALID_ARG, "k_prefix.len_s != v_prefix.len_s");
  if (ks->len_s != vs->len_s) return fail(SK_ERR_INVALID_ARG, "k_suffix.len_s != v_suffix.len_s");
  const int64_t Sp = kp->len_s, Ss = ks->len_s, Skv = Sp + Ss;
  if (Skv > INT32_MAX) return fail(SK_ERR_INVALID_ARG, "Sp + Ss too large");
  if (!scatter && !no_self_overlap(*out, B, Hq, D)) return fail(SK_ERR_INVALID_ARG, "out overlaps itself");
  if (B == 0 || Sq == 0) return SK_OK;
  if (!scatter) {  // destinations of a scattered output may live on other GPUs: the caller keeps them apart
    Span so, si;
    span_of(*out, B, Hq, D, &so);
    const struct { const char* n; const sk_tensor_t* t; int H; } ins[5] = {
        {"q", q, Hq}, {"k_prefix", kp, Hkv}, {"v_prefix", vp, Hkv}, {"k_suffix", ks, Hkv}, {"v_suffix", vs, Hkv}};
    for (auto& in : ins) {
      span_of(*in.t, B, in.H, D, &si);
      if (overlaps(so, si)) return fail(SK_ERR_INVALID_ARG, "out overlaps %s", in.n);
    }
  }
  for (int b = 0; b < B; ++b) {
    const int64_t n = real_len ? real_len[b] : Skv;
    if (n < 0 || n > Skv) return fail(SK_ERR_INVALID_ARG, "real_len[%d]=%lld outside [0, %lld]", b, (long long)n, (long long)Skv);
    if (q_valid_in && (q_valid_in[b] < 0 || q_valid_in[b] > Sq))
      return fail(SK_ERR_INVALID_ARG, "q_valid[%d]=%d outside [0, %d]", b, q_valid_in[b], Sq);
  }

  int dev = 0;
  DeviceInfo* info = nullptr;
  if ((st = device_setup(&dev, &info)) != SK_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);

  const int n_qtiles = (Sq + skattn::kRowsPerCta - 1) / skattn::kRowsPerCta;
  for (int b0 = 0; b0 < B; b0 += skattn::kMaxBatch) {
    const int nb = std::min(skattn::kMaxBatch, B - b0);
    skattn::AttnParams prm;
    std::memset(&prm, 0, sizeof prm);
    for (int i = 0; i < nb; ++i) {
      const int b = b0 + i;
      const int64_t n = real_len ? real_len[b] : Skv;
      const int64_t npre = std::min<int64_t>(Sp, n);
      const int64_t nsuf = std::max<int64_t>(0, n - Sp);
      // joint self-attention (Sq == Skv): the tail pad covers the query stream too
      const int64_t qv = q_valid_in ? q_valid_in[b] : (Sq == Skv ? n : Sq);
      prm.q_valid[i] = static_cast<int32_t>(qv);
      prm.n_prefix[i] = static_cast<int32_t>(npre);
      prm.n_suffix[i] = static_cast<int32_t>(nsuf);
      prm.sq[i] = Sq;
      prm.out_off[i] = static_cast<int64_t>(i) * out->stride_b;
      auto bptr = [&](const sk_tensor_t* t) {
        return static_cast<const void*>(static_cast<const uint16_t*>(t->ptr) + static_cast<int64_t>(b) * t->stride_b);
      };
      if (qv > 0 && n > 0)
        if ((st = encode_map(&prm.tm_q[i], bptr(q), q->stride_s, q->stride_h, Hq, qv, D)) != SK_OK) return st;
      if (npre > 0) {
        if ((st = encode_map(&prm.tm_kp[i], bptr(kp), kp->stride_s, kp->stride_h, Hkv, npre, D)) != SK_OK) return st;
        if ((st = encode_map(&prm.tm_vp[i], bptr(vp), vp->stride_s, vp->stride_h, Hkv, npre, D)) != SK_OK) return st;
      }
      if (nsuf > 0) {
        if ((st = encode_map(&prm.tm_ks[i], bptr(ks), ks->stride_s, ks->stride_h, Hkv, nsuf, D)) != SK_OK) return st;
        if ((st = encode_map(&prm.tm_vs[i], bptr(vs), vs->stride_s, vs->stride_h, Hkv, nsuf, D)) != SK_OK) return st;
      }
    }
    prm.out_ss = out->stride_s;
    prm.out_sh = out->stride_h;
    if (scatter) {
      prm.out_chunk = out->len_s;
      for (int r = 0; r < scatter->n; ++r)
        prm.out_dst[r] = static_cast<uint16_t*>(scatter->dst[r]) + static_cast<int64_t>(b0) * out->stride_b +
                         static_cast<int64_t>(scatter->head_offset) * out->stride_h;
    } else {
      prm.out = static_cast<uint16_t*>(out->ptr) + static_cast<int64_t>(b0) * out->stride_b;
    }
    prm.group = Hq / Hkv;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.status = info->status;
    prm.wait_limit_ns = g_wait_limit_ns;
    prm.test_stall = g_test_stall;
    st = (D == 64) ? launch_attn<64>(prm, n_qtiles, Hq, nb, stream, info)
                   : launch_attn<128>(prm, n_qtiles, Hq, nb, stream, info);
    if (st != SK_OK) return st;
  }
  return SK_OK;
}

// Packed varlen input on the persistent kernel: one tensor map per packed
// tensor, the segments' rows and lengths in the launch parameters, segments
// processed longest first (a static schedule over the SMs balances best when
// the big units come first); one launch per kMaxSegments segments.
template <int D>
sk_status_t launch_varlen(skattn::VarlenParams& prm, cudaStream_t stream, DeviceInfo* dev) {
  using L = skattn::PSmemLayout<D>;
  const int slot = 4 + (D == 64 ? 0 : 1);
  auto kernel = skattn::attn_fwd_persistent_kernel<D, false, skattn::VarlenParams>;
  sk_status_t st;
  if ((st = set_smem<D>(reinterpret_cast<const void*>(kernel), slot, L::kAlloc, dev, skattn::kLaunchRegs)) != SK_OK)
    return st;
  const int grid = std::min(prm.n_units, dev->sm_count);
  kernel<<<grid, skattn::kPThreads, L::kAlloc, stream>>>(prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch (packed)");
  return SK_OK;
}

sk_status_t varlen_persistent(const sk_tensor_t* q, const sk_tensor_t* k, const sk_tensor_t* v,
                              const int32_t* cu_q, const int32_t* cu_k, const int32_t* used_q,
                              const int32_t* used_k, int32_t nseg, int32_t Hq, int32_t Hkv, float scale,
                              const sk_tensor_t* out, int32_t D, cudaStream_t stream, DeviceInfo* info) {
  struct Seg { int32_t q0, k0, lq, qv, nk; int64_t cost; };
  std::vector<Seg> segs;
  segs.reserve(nseg);
  bool any_q = false, any_k = false;
  for (int i = 0; i < nseg; ++i) {
    Seg g;
    g.q0 = cu_q[i];
    g.k0 = cu_k[i];
    g.lq = cu_q[i + 1] - cu_q[i];
    g.qv = used_q ? used_q[i] : g.lq;
    g.nk = used_k ? used_k[i] : cu_k[i + 1] - cu_k[i];
    if (g.lq == 0) continue;  // no rows: nothing to write
    const int64_t pairs = (g.lq + skattn::kRowsPerCta - 1) / skattn::kRowsPerCta;
    const int64_t tiles = (g.nk + skattn::kBlockN - 1) / skattn::kBlockN;
    g.cost = pairs * std::max<int64_t>(tiles, 1);
    any_q = any_q || (g.qv > 0 && g.nk > 0);
    any_k = any_k || g.nk > 0;
    segs.push_back(g);
  }
  std::stable_sort(segs.begin(), segs.end(), [](const Seg& a, const Seg& b) { return a.cost > b.cost; });
  static thread_local skattn::VarlenParams prm;
  std::memset(static_cast<void*>(&prm), 0, offsetof(skattn::VarlenParams, seg_unit0));
  sk_status_t st;
  if (any_q && any_k) {
    if ((st = encode_map(&prm.tm_q, q->ptr, q->stride_s, q->stride_h, Hq, q->len_s, D)) != SK_OK) return st;
    if ((st = encode_map(&prm.tm_k, k->ptr, k->stride_s, k->stride_h, Hkv, k->len_s, D)) != SK_OK) return st;
    if ((st = encode_map(&prm.tm_v, v->ptr, v->stride_s, v->stride_h, Hkv, v->len_s, D)) != SK_OK) return st;
  }
  prm.out = static_cast<uint16_t*>(out->ptr);
  prm.out_ss = out->stride_s;
  prm.out_sh = out->stride_h;
  prm.n_heads = Hq;
  prm.group = Hq / Hkv;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.status = info->status;
  prm.wait_limit_ns = g_wait_limit_ns;
  prm.test_stall = g_test_stall;
  for (size_t s0 = 0; s0 < segs.size(); s0 += skattn::kMaxSegments) {
    const int n = static_cast<int>(std::min<size_t>(skattn::kMaxSegments, segs.size() - s0));
    int64_t units = 0;
    for (int i = 0; i < n; ++i) {
      const Seg& g = segs[s0 + i];
      if (units > INT32_MAX) return fail(SK_ERR_UNSUPPORTED, "too many work units");
      prm.seg_unit0[i] = static_cast<int32_t>(units);
      prm.seg_q0[i] = g.q0;
      prm.seg_k0[i] = g.k0;
      prm.seg_lq[i] = g.lq;
      prm.seg_qv[i] = g.qv;
      prm.seg_nk[i] = g.nk;
      units += static_cast<int64_t>(Hq) * ((g.lq + skattn::kRowsPerCta - 1) / skattn::kRowsPerCta);
    }
    if (units > INT32_MAX) return fail(SK_ERR_UNSUPPORTED, "too many work units");
    prm.n_seg = n;
    prm.n_units = static_cast<int32_t>(units);
    st = (D == 64) ? launch_varlen<64>(prm, stream, info) : launch_varlen<128>(prm, stream, info);
    if (st != SK_OK) return st;
  }
  return SK_OK;
}

// Packed varlen input: segment i owns query rows [cu_q[i], cu_q[i+1]) and key
// rows [cu_k[i], cu_k[i+1]) of single-row tensors.  Validation here; the launch
// (varlen_persistent) uses one tensor map per packed tensor and passes each
// segment's first rows and lengths in the launch parameters, so the
// block-diagonal mask costs nothing: a unit only ever loads its own segment's
// rows.
sk_status_t varlen_impl(const sk_tensor_t* q, const sk_tensor_t* k, const sk_tensor_t* v,
                        const int32_t* cu_q, const int32_t* cu_k, const int32_t* used_q,
                        const int32_t* used_k, int32_t nseg, int32_t Hq, int32_t Hkv, float scale,
                        const sk_tensor_t* out, int32_t D, void* stream_v) {
  if (nseg < 0) return fail(SK_ERR_INVALID_ARG, "num_segments < 0");
  if (nseg > 0 && (!cu_q || !cu_k)) return fail(SK_ERR_INVALID_ARG, "cu_seqlens arrays are NULL");
  if (Hq <= 0 || Hkv <= 0) return fail(SK_ERR_INVALID_ARG, "head counts must be positive");
  if (Hq % Hkv != 0) return fail(SK_ERR_INVALID_ARG, "num_q_heads %% num_kv_heads != 0");
  if (Hq > 65535) return fail(SK_ERR_UNSUPPORTED, "num_q_heads > 65535");
  if (D != 64 && D != 128) return fail(SK_ERR_UNSUPPORTED, "head_dim %d not in {64, 128}", D);
  if (!(std::isfinite(scale) && scale >= 0.f)) return fail(SK_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  sk_status_t st;
  if ((st = check_tensor("q", q, 1, Hq, D)) != SK_OK) return st;
  if ((st = check_tensor("k", k, 1, Hkv, D)) != SK_OK) return st;
  if ((st = check_tensor("v", v, 1, Hkv, D)) != SK_OK) return st;
  if ((st = check_tensor("out", out, 1, Hq, D)) != SK_OK) return st;
  if (out->len_s != q->len_s) return fail(SK_ERR_INVALID_ARG, "out.len_s (%d) != q.len_s (%d)", out->len_s, q->len_s);
  if (k->len_s != v->len_s) return fail(SK_ERR_INVALID_ARG, "k.len_s != v.len_s");
  if (!no_self_overlap(*out, 1, Hq, D)) return fail(SK_ERR_INVALID_ARG, "out overlaps itself");
  if (nseg == 0) return SK_OK;
  if (cu_q[0] < 0 || cu_k[0] < 0) return fail(SK_ERR_INVALID_ARG, "cu_seqlens[0] < 0");
  int32_t max_sq = 0;
  for (int i = 0; i < nseg; ++i) {
    const int64_t lq = static_cast<int64_t>(cu_q[i + 1]) - cu_q[i];
    const int64_t lk = static_cast<int64_t>(cu_k[i + 1]) - cu_k[i];
    if (lq < 0 || lk < 0) return fail(SK_ERR_INVALID_ARG, "cu_seqlens decrease at segment %d", i);
    if (used_q && (used_q[i] < 0 || used_q[i] > lq))
      return fail(SK_ERR_INVALID_ARG, "seqused_q[%d]=%d outside [0, %lld]", i, used_q[i], (long long)lq);
    if (used_k && (used_k[i] < 0 || used_k[i] > lk))
      return fail(SK_ERR_INVALID_ARG, "seqused_k[%d]=%d outside [0, %lld]", i, used_k[i], (long long)lk);
    max_sq = std::max<int32_t>(max_sq, static_cast<int32_t>(lq));
  }
  if (cu_q[nseg] > q->len_s) return fail(SK_ERR_INVALID_ARG, "cu_seqlens_q[%d]=%d > q.len_s=%d", nseg, cu_q[nseg], q->len_s);
  if (cu_k[nseg] > k->len_s) return fail(SK_ERR_INVALID_ARG, "cu_seqlens_k[%d]=%d > k.len_s=%d", nseg, cu_k[nseg], k->len_s);
  if (max_sq == 0) return SK_OK;
  Span so, si;
  span_of(*out, 1, Hq, D, &so);
  const struct { const char* n; const sk_tensor_t* t; int H; } ins[3] = {{"q", q, Hq}, {"k", k, Hkv}, {"v", v, Hkv}};
  for (auto& in : ins) {
    span_of(*in.t, 1, in.H, D, &si);
    if (overlaps(so, si)) return fail(SK_ERR_INVALID_ARG, "out overlaps %s", in.n);
  }

  int dev = 0;
  DeviceInfo* info = nullptr;
  if ((st = device_setup(&dev, &info)) != SK_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  return varlen_persistent(q, k, v, cu_q, cu_k, used_q, used_k, nseg, Hq, Hkv, scale, out, D, stream, info);
}

}  // namespace

extern "C" {

sk_status_t attn_fwd_split_kv(const sk_tensor_t* q, const sk_tensor_t* k_prefix, const sk_tensor_t* v_prefix,
                              const sk_tensor_t* k_suffix, const sk_tensor_t* v_suffix, const int32_t* real_len,
                              int32_t num_q_heads, int32_t num_kv_heads, float softmax_scale,
                              const sk_tensor_t* out, int32_t batch, int32_t head_dim, void* stream) {
  try {
    return attn_impl(q, k_prefix, v_prefix, k_suffix, v_suffix, real_len, num_q_heads, num_kv_heads,
                     softmax_scale, out, batch, head_dim, nullptr, stream);
  } catch (...) {
    return fail(SK_ERR_INVALID_ARG, "internal exception");
  }
}

sk_status_t attn_fwd_split_kv_scatter(const sk_tensor_t* q, const sk_tensor_t* k_prefix,
                                      const sk_tensor_t* v_prefix, const sk_tensor_t* k_suffix,
                                      const sk_tensor_t* v_suffix, const int32_t* real_len,
                                      const int32_t* q_valid, int32_t num_q_heads, int32_t num_kv_heads,
                                      float softmax_scale, void* const* dst, int32_t num_dst,
                                      const sk_tensor_t* dst_layout, int32_t head_offset, int32_t batch,
                                      int32_t head_dim, void* stream) {
  try {
    const ScatterOut sc{dst, num_dst, dst_layout, head_offset};
    return attn_impl(q, k_prefix, v_prefix, k_suffix, v_suffix, real_len, num_q_heads, num_kv_heads,
                     softmax_scale, nullptr, batch, head_dim, q_valid, stream, &sc);
  } catch (...) {
    return fail(SK_ERR_INVALID_ARG, "internal exception");
  }
}

sk_status_t attn_fwd_split_kv_ex(const sk_tensor_t* q, const sk_tensor_t* k_prefix,
                                 const sk_tensor_t* v_prefix, const sk_tensor_t* k_suffix,
                                 const sk_tensor_t* v_suffix, const int32_t* real_len,
                                 int32_t num_q_heads, int32_t num_kv_heads, float softmax_scale,
                                 const sk_tensor_t* out, int32_t batch, int32_t head_dim,
                                 const int32_t* q_valid, void* stream) {
  try {
    return attn_impl(q, k_prefix, v_prefix, k_suffix, v_suffix, real_len, num_q_heads, num_kv_heads,
                     softmax_scale, out, batch, head_dim, q_valid, stream);
  } catch (...) {
    return fail(SK_ERR_INVALID_ARG, "internal exception");
  }
}

sk_status_t attn_fwd_varlen(const sk_tensor_t* q, const sk_tensor_t* k, const sk_tensor_t* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            const int32_t* seqused_q, const int32_t* seqused_k, int32_t num_segments,
                            int32_t num_q_heads, int32_t num_kv_heads, float softmax_scale,
                            const sk_tensor_t* out, int32_t head_dim, void* stream) {
  try {
    return varlen_impl(q, k, v, cu_seqlens_q, cu_seqlens_k, seqused_q, seqused_k, num_segments,
                       num_q_heads, num_kv_heads, softmax_scale, out, head_dim, stream);
  } catch (...) {
    return fail(SK_ERR_INVALID_ARG, "internal exception");
  }
}

sk_status_t sk_shard_pad_copy(const void* src, int64_t src_stride_b, int64_t src_stride_s, int32_t src_rows,
                              void* dst, int64_t dst_stride_b, int64_t dst_stride_s, int32_t dst_rows,
                              int32_t first_row, int32_t row_bytes, int32_t batch, int32_t pad_mode,
                              void* stream) {
  try {
    if (batch < 0 || src_rows < 0 || dst_rows < 0 || first_row < 0)
      return fail(SK_ERR_INVALID_ARG, "negative size");
    if (row_bytes <= 0 || row_bytes % 16 != 0) return fail(SK_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 16");
    if (pad_mode != 0 && pad_mode != 1) return fail(SK_ERR_INVALID_ARG, "pad_mode must be 0 (zeros) or 1 (repeat last)");
    if (pad_mode == 1 && src_rows == 0 && dst_rows > 0) return fail(SK_ERR_INVALID_ARG, "repeat_last needs a source row");
    if (batch == 0 || dst_rows == 0) return SK_OK;
    const int64_t st[4] = {src_stride_b, src_stride_s, dst_stride_b, dst_stride_s};
    for (int64_t v : st)
      if (v < 0 || v % 16 != 0) return fail(SK_ERR_INVALID_ARG, "strides must be non-negative multiples of 16 bytes");
    if (!dst || (src_rows > 0 && !src)) return fail(SK_ERR_INVALID_ARG, "NULL pointer");
    if (reinterpret_cast<uintptr_t>(dst) % 16 || reinterpret_cast<uintptr_t>(src) % 16)
      return fail(SK_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if (dst_stride_s < row_bytes) return fail(SK_ERR_INVALID_ARG, "dst rows overlap");
    if (batch > 1 && dst_stride_b < static_cast<int64_t>(dst_rows) * dst_stride_s)
      return fail(SK_ERR_INVALID_ARG, "dst batch rows overlap");
    // destination must not overlap the source rows it reads
    if (src_rows > 0) {
      const uintptr_t d0 = reinterpret_cast<uintptr_t>(dst);
      const uintptr_t d1 = d0 + static_cast<uintptr_t>((batch - 1) * dst_stride_b + (dst_rows - 1) * dst_stride_s + row_bytes);
      const uintptr_t s0 = reinterpret_cast<uintptr_t>(src);
      const uintptr_t s1 = s0 + static_cast<uintptr_t>((batch - 1) * src_stride_b + (src_rows - 1) * src_stride_s + row_bytes);
      if (d0 < s1 && s0 < d1) return fail(SK_ERR_INVALID_ARG, "dst overlaps src");
    }
    int dev = 0;
    DeviceInfo* info = nullptr;
    sk_status_t stt;
    if ((stt = device_setup(&dev, &info)) != SK_OK) return stt;
    skshard::PadCopyParams prm;
    prm.src = static_cast<const uint8_t*>(src);
    prm.dst = static_cast<uint8_t*>(dst);
    prm.src_sb = src_stride_b;
    prm.src_ss = src_stride_s;
    prm.dst_sb = dst_stride_b;
    prm.dst_ss = dst_stride_s;
    prm.src_rows = src_rows;
    prm.dst_rows = dst_rows;
    prm.first_row = first_row;
    prm.row_chunks = row_bytes / 16;
    prm.batch = batch;
    prm.repeat_last = pad_mode;
    const int64_t total = static_cast<int64_t>(batch) * dst_rows * prm.row_chunks;
    const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, int64_t(info->sm_count) * 8));
    skshard::pad_copy_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(prm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pad_copy_kernel launch");
    return SK_OK;
  } catch (...) {
    return fail(SK_ERR_INVALID_ARG, "internal exception");
  }
}

sk_status_t qk_rmsnorm_rope(const sk_tensor_t* q, const sk_tensor_t* k, const void* w_q, const void* w_k,
                            const float* rope_table, int32_t table_rows, int32_t rot_dim,
                            int32_t interleaved, float eps, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t batch, int32_t head_dim, int32_t exact, void* stream) {
  try {
    if (batch < 0) return fail(SK_ERR_INVALID_ARG, "batch < 0");
    if (num_q_heads <= 0 || num_kv_heads <= 0) return fail(SK_ERR_INVALID_ARG, "head counts must be positive");
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
      return fail(SK_ERR_UNSUPPORTED, "head_dim %d not in {64, 128, 256}", head_dim);
    if (rot_dim < 0 || rot_dim > head_dim || (rot_dim & 1)) return fail(SK_ERR_INVALID_ARG, "rot_dim must be even and in [0, head_dim]");
    if (!(std::isfinite(eps) && eps >= 0.f)) return fail(SK_ERR_INVALID_ARG, "eps must be finite and >= 0");
    sk_status_t st;
    if ((st = check_tensor("q", q, batch, num_q_heads, head_dim)) != SK_OK) return st;
    if ((st = check_tensor("k", k, batch, num_kv_heads, head_dim)) != SK_OK) return st;
    if (q->len_s != k->len_s) return fail(SK_ERR_INVALID_ARG, "q.len_s != k.len_s");
    const int32_t S = q->len_s;
    if (batch == 0 || S == 0) return SK_OK;
    if (!no_self_overlap(*q, batch, num_q_heads, head_dim) || !no_self_overlap(*k, batch, num_kv_heads, head_dim))
      return fail(SK_ERR_INVALID_ARG, "q or k overlaps itself");
    Span sq, sk;
    span_of(*q, batch, num_q_heads, head_dim, &sq);
    span_of(*k, batch, num_kv_heads, head_dim, &sk);
    if (overlaps(sq, sk)) {
      // Allowed only for head ranges of one fused buffer: same strides, k's
      // first head m whole heads after q's (m >= Hq), and the layout with
      // m + Hkv heads free of self-overlap, so no element is both a q and a k
      // element (k shifted by a token, or heads spilling into the next
      // token, are rejected).
      const int64_t off = (static_cast<const uint16_t*>(k->ptr) - static_cast<const uint16_t*>(q->ptr));
      bool fused = q->stride_b == k->stride_b && q->stride_s == k->stride_s && q->stride_h == k->stride_h &&
                   q->stride_h > 0 && off >= 0 && off % q->stride_h == 0 && off / q->stride_h >= num_q_heads;
      if (fused) {
        const int64_t m = off / q->stride_h;
        fused = m + num_kv_heads <= INT32_MAX &&
                no_self_overlap(*q, batch, static_cast<int>(m + num_kv_heads), head_dim);
      }
      if (!fused) return fail(SK_ERR_INVALID_ARG, "q and k overlap");
    }
    if (!w_q || !w_k || (rot_dim > 0 && !rope_table)) return fail(SK_ERR_INVALID_ARG, "NULL weight or table");
    if (reinterpret_cast<uintptr_t>(w_q) % 16 || reinterpret_cast<uintptr_t>(w_k) % 16 ||
        reinterpret_cast<uintptr_t>(rope_table) % 16)
      return fail(SK_ERR_INVALID_ARG, "weights and table must be 16-byte aligned");
    if (rot_dim > 0 && table_rows < S) return fail(SK_ERR_INVALID_ARG, "table_rows < seq len");
    if (interleaved && rot_dim % 8 != 0)
      return fail(SK_ERR_UNSUPPORTED, "interleaved rot_dim must be a multiple of 8");
    if (!interleaved && rot_dim % 16 != 0)
      return fail(SK_ERR_UNSUPPORTED, "half-split rot_dim must be a multiple of 16");
    int dev = 0;
    DeviceInfo* info = nullptr;
    if ((st = device_setup(&dev, &info)) != SK_OK) return st;
    skqkn::NormRopeParams prm;
    prm.q = static_cast<uint16_t*>(q->ptr);
    prm.k = static_cast<uint16_t*>(k->ptr);
    prm.q_sb = q->stride_b; prm.q_ss = q->stride_s; prm.q_sh = q->stride_h;
    prm.k_sb = k->stride_b; prm.k_ss = k->stride_s; prm.k_sh = k->stride_h;
    prm.w_q = static_cast<const uint16_t*>(w_q);
    prm.w_k = static_cast<const uint16_t*>(w_k);
    prm.table = rope_table;
    prm.rot_dim = rot_dim;
    prm.interleaved = interleaved != 0;
    prm.eps = eps;
    prm.S = S;
    prm.Hq = num_q_heads;
    prm.Hkv = num_kv_heads;
    prm.B = batch;
    cudaError_t e = skqkn::launch(prm, head_dim, exact != 0, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "qk_rmsnorm_rope launch");
    return SK_OK;
  } catch (...) {
    return fail(SK_ERR_INVALID_ARG, "internal exception");
  }
}

const char* sk_last_error(void) { return g_last_error.c_str(); }

sk_status_t sk_device_status(int32_t device, int32_t* status_out, int32_t clear) {
  if (!status_out) return fail(SK_ERR_INVALID_ARG, "status_out is NULL");
  int prev = 0;
  cudaError_t e = cudaGetDevice(&prev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (device != prev && (e = cudaSetDevice(device)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  sk_status_t st = SK_OK;
  int32_t v = 0;
  e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof v);
  if (e == cudaSuccess && clear) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero);
  }
  if (e != cudaSuccess) st = cuda_fail(e, "reading device status");
  *status_out = v;
  if (device != prev) cudaSetDevice(prev);
  return st;
}

sk_status_t sk_set_wait_timeout_ms(int32_t ms) {
  if (ms < 1 || ms > 60000) return fail(SK_ERR_INVALID_ARG, "timeout must be in [1, 60000] ms");
  std::lock_guard<std::mutex> lk(g_mu);
  g_wait_limit_ns = static_cast<uint64_t>(ms) * 1000000ull;
  return SK_OK;
}

sk_status_t sk_test_stall_mma(int32_t on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_test_stall = on ? 1 : 0;
  return SK_OK;
}

int32_t sk_abi_version(void) { return kAbiVersion; }

}  // extern "C"
