// Split-KV tail-padded attention forward for sm_100a: persistent CTAs, the
// probabilities P kept in tensor memory.
//
//   O = softmax(scale * Q K*^T) V*,  K*/V* = cat(prefix, suffix)[0:real_len]
// ("sglang PR 26973", forward_with_replicated_kv_prefix; "sglang PR 30107",
// tail_attn_meta / tail-pad layout invariant).  The concatenation is never
// built: the KV tile loop walks the prefix tensor map, then the suffix one,
// each clipped on the host to the valid keys of its batch row, so no pad byte
// is fetched (rows past a map's extent arrive as zeros) and tiles past
// real_len are never issued; the one partial tile of each source is masked
// column-wise.
//
// Work: a unit is 256 consecutive query rows (two 128-row tiles A and B) of
// one (entry, query head); an entry is a batch row or a packed segment.  One
// CTA per SM walks units blockIdx.x, blockIdx.x + gridDim.x, ...  All
// barrier phases and the K/V rings run on across units, so the next unit's
// Q load and first score MMAs overlap the previous unit's last PV MMAs and
// epilogue.
//
// Warp roles (384 threads):
//   warps 0-3  tile A, warps 4-7 tile B: thread t of a warpgroup owns query
//              row t of its tile (TMEM lane t): loads its score row from
//              TMEM, online softmax in fp32 (exp2, scale*log2 e folded in,
//              running max raised only past kRescaleLog2, then O rescaled in
//              TMEM), writes P as bf16 pairs back over the first 64 columns
//              of its own score row, and at the end of a unit reads O, divides
//              by the row sum and stores the bf16 row.  After a unit's first
//              tile the row is loaded in two halves and the first half's
//              exponentials run on the running max while the second half
//              arrives; the tile's max is checked before any key is released.
//   warp 8     TMA producer: Q tiles per unit, K and V tiles into rings.
//   warp 9     TMEM allocator and tcgen05.mma issuer.  Per KV tile j the
//              order is PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), each PV in two
//              halves (keys 0-63 once the softmax has released them, then
//              keys 64-127): PV takes P from TMEM (A operand) and V from
//              shared memory, so only K, V and Q are read from shared memory.
//              S_X(j+1) overwrites the columns PV_X(j) reads P from; it is
//              issued behind PV_X(j) on the same in-order MMA pipe, with no
//              wait in between.
//   warps 10-11 idle (they complete the third warpgroup, whose registers go
//              to the softmax warpgroups).
// TMEM (512 columns): S_A/P_A [0,128), S_B/P_B [128,256), O_A [256,256+D),
// O_B [384,384+D).
// Every wait is bounded (globaltimer); on expiry the CTA raises the device
// status word, drains its own copies and MMAs, frees TMEM and exits.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "attn_common.cuh"
#include "ptx.cuh"

namespace skattn {

// 12 warps: 0-3 tile A, 4-7 tile B, 8 TMA, 9 MMA, 10-11 idle (they complete
// warpgroup 2, which gives registers back).  Launched at kLaunchRegs per
// thread; the softmax warpgroups then raise to kSoftmaxRegs and warpgroup 2
// lowers to kOtherRegs: 2 * 128 * 224 + 128 * 56 = 384 * 168, the launch's
// allocation exactly.  The host launches only when the compiled kernel uses
// kLaunchRegs registers (a smaller launch allocation would leave the raise
// waiting for registers that never come).
constexpr int kPThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kOtherRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kPThreads * kLaunchRegs, "register split");

template <int D>
struct PSmemLayout {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr uint32_t kSub = kBlockM * 128;  // one 64-column (128 B) swizzled sub-tile
  static constexpr uint32_t kQTile = kBlockM * D * 2;
  static constexpr uint32_t kKVTile = kBlockN * D * 2;
  static constexpr int kKS = D == 128 ? 3 : 4;  // K ring depth
  static constexpr int kVS = D == 128 ? 2 : 4;  // V ring depth
  static constexpr uint32_t kQ = 0;                              // + tile * kQTile
  static constexpr uint32_t kK = kQ + kTilesPerCta * kQTile;     // + stage * kKVTile
  static constexpr uint32_t kV = kK + kKS * kKVTile;             // + stage * kKVTile
  static constexpr uint32_t kBar = kV + kVS * kKVTile;
  static constexpr int bQFull = 0;                  // + tile
  static constexpr int bQEmpty = bQFull + 2;        // + tile: S_X(last) of the unit finished
  static constexpr int bKFull = bQEmpty + 2;        // + stage
  static constexpr int bKEmpty = bKFull + kKS;      // + stage
  static constexpr int bVFull = bKEmpty + kKS;      // + stage
  static constexpr int bVEmpty = bVFull + kVS;      // + stage
  static constexpr int bSFull = bVEmpty + kVS;      // + tile: S_X(j) is in TMEM
  static constexpr int bPLo = bSFull + 2;           // + tile: P_X(j) keys 0-63 in TMEM (128 arrivals)
  static constexpr int bPHi = bPLo + 2;             // + tile: P_X(j) keys 64-127 in TMEM (128 arrivals)
  static constexpr int bOFull = bPHi + 2;           // + tile: PV_X(last) of the unit finished
  static constexpr int bMmaDone = bOFull + 2;
  static constexpr int kNumBars = bMmaDone + 1;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kEnd = kMisc + 16;
  static constexpr uint32_t kAlloc = (kEnd + 1024) > 120 * 1024 ? (kEnd + 1024) : 120 * 1024;
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

// Packed variable-length input: segments of one packed Q [Tq] and K/V [Tk]
// token axis, each attending only to its own keys.  One tensor map per packed
// tensor; per segment its first rows, lengths and first work unit (segments
// are listed in processing order, longest first, and unit u belongs to the
// last segment whose first unit is <= u).
constexpr int kMaxSegments = 1024;

struct alignas(64) VarlenParams {
  CUtensorMap tm_q, tm_k, tm_v;
  uint16_t* out;
  int64_t out_ss, out_sh;
  int32_t n_seg;                // segments with at least one unit
  int32_t n_heads;              // query heads
  int32_t n_units;              // sum over segments of n_heads * ceil(len_q / 256)
  int32_t group;                // num_q_heads / num_kv_heads
  float scale_log2;             // softmax_scale * log2(e)
  int32_t* status;              // device status word
  uint64_t wait_limit_ns;
  int32_t test_stall;
  int32_t seg_unit0[kMaxSegments];  // first unit of the segment
  int32_t seg_q0[kMaxSegments];     // first row of the segment in q / out
  int32_t seg_k0[kMaxSegments];     // first row of the segment in k / v
  int32_t seg_lq[kMaxSegments];     // query rows (rows in [seg_qv, seg_lq) are pad: zeros)
  int32_t seg_qv[kMaxSegments];     // valid query rows
  int32_t seg_nk[kMaxSegments];     // valid keys
};

// One unit of work: query rows [row0, row0 + 256) of entry bl (a batch row or
// a segment), query head hq.  Rows and keys are counted from q_off / k_off
// in the tensors the maps describe (0 for a batch row: its maps start there).
struct PUnit {
  int bl, hq, row0, qv, sq, nkp, nks, tP, n_tiles, q_off, k_off;
  bool compute;  // false: no valid query row or no valid key (rows written as zeros, if any)
};

__device__ __forceinline__ PUnit decode_unit(const AttnParams& p, int u) {
  PUnit t;
  const int pair = u % p.n_pairs;
  const int rest = u / p.n_pairs;
  t.hq = rest % p.n_heads;
  t.bl = rest / p.n_heads;
  t.row0 = pair * kRowsPerCta;
  t.qv = p.q_valid[t.bl];
  t.sq = p.sq[t.bl];
  t.nkp = p.n_prefix[t.bl];
  t.nks = p.n_suffix[t.bl];
  t.tP = (t.nkp + kBlockN - 1) / kBlockN;
  t.n_tiles = t.tP + (t.nks + kBlockN - 1) / kBlockN;
  t.q_off = 0;
  t.k_off = 0;
  t.compute = t.row0 < t.qv && t.n_tiles > 0;
  return t;
}

__device__ __forceinline__ PUnit decode_unit(const VarlenParams& p, int u) {
  int lo = 0, hi = p.n_seg - 1;  // last segment with seg_unit0 <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (p.seg_unit0[mid] <= u) lo = mid; else hi = mid - 1;
  }
  PUnit t;
  const int s = lo;
  const int lq = p.seg_lq[s];
  const int pairs = (lq + kRowsPerCta - 1) / kRowsPerCta;
  const int v = u - p.seg_unit0[s];
  t.bl = s;
  t.hq = v / pairs;
  t.row0 = (v % pairs) * kRowsPerCta;
  t.qv = p.seg_qv[s];
  t.sq = lq;
  t.nkp = 0;
  t.nks = p.seg_nk[s];
  t.tP = 0;
  t.n_tiles = (t.nks + kBlockN - 1) / kBlockN;
  t.q_off = p.seg_q0[s];
  t.k_off = p.seg_k0[s];
  t.compute = t.row0 < t.qv && t.n_tiles > 0;
  return t;
}

__device__ __forceinline__ const CUtensorMap* q_map(const AttnParams& p, const PUnit& t) { return &p.tm_q[t.bl]; }
__device__ __forceinline__ const CUtensorMap* k_map(const AttnParams& p, const PUnit& t, bool pre) {
  return pre ? &p.tm_kp[t.bl] : &p.tm_ks[t.bl];
}
__device__ __forceinline__ const CUtensorMap* v_map(const AttnParams& p, const PUnit& t, bool pre) {
  return pre ? &p.tm_vp[t.bl] : &p.tm_vs[t.bl];
}
__device__ __forceinline__ const CUtensorMap* q_map(const VarlenParams& p, const PUnit&) { return &p.tm_q; }
__device__ __forceinline__ const CUtensorMap* k_map(const VarlenParams& p, const PUnit&, bool) { return &p.tm_k; }
__device__ __forceinline__ const CUtensorMap* v_map(const VarlenParams& p, const PUnit&, bool) { return &p.tm_v; }

template <bool kScatter>
__device__ __forceinline__ uint16_t* unit_row_ptr(const AttnParams& p, const PUnit& t, int row) {
  return out_row_ptr<kScatter>(p, t.bl, t.hq, row);
}
template <bool kScatter>
__device__ __forceinline__ uint16_t* unit_row_ptr(const VarlenParams& p, const PUnit& t, int row) {
  return p.out + static_cast<int64_t>(t.q_off + row) * p.out_ss + static_cast<int64_t>(t.hq) * p.out_sh;
}

// Maximum of 64 scores s[B .. B + 63]: two chains of three-input maxima.
template <int B>
__device__ __forceinline__ float half_max(const float (&s)[kBlockN]) {
  float mx[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    mx[k] = fmaxf(s[B + k], s[B + k + 2]);
#pragma unroll
    for (int c = B + 4 + k; c < B + 64; c += 4) mx[k] = skptx::fmax3(mx[k], s[c], s[c + 2]);
  }
  return fmaxf(mx[0], mx[1]);
}

// Columns [32 * C, 32 * C + 32) of one score row (already masked) -> 16 bf16
// pairs of p = 2^(s * sl2 - m) in pk, their fp32 sum added to acc.  Masked
// columns (partial tile) are exact zeros.
template <bool kPartial, int C, int N>
__device__ __forceinline__ void exp_chunk(const float (&s)[N], uint64_t sl2_2, uint64_t negm_2, int nvalid,
                                          uint32_t (&pk)[16], uint64_t (&acc)[4]) {
  static_assert(32 * C + 32 <= N, "chunk inside the row");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = C * 32 + 2 * i;
    const uint64_t x = skptx::fma2(skptx::f2_pack(s[c], s[c + 1]), sl2_2, negm_2);
    float x0, x1;
    skptx::f2_unpack(x, x0, x1);
    float e0 = skptx::ex2_approx(x0);
    float e1 = skptx::ex2_approx(x1);
    // exact zeros for masked columns (also when scale == 0: -inf * 0 is NaN)
    if (kPartial && c >= nvalid) e0 = 0.f;
    if (kPartial && c + 1 >= nvalid) e1 = 0.f;
    acc[i % 4] = skptx::add2(acc[i % 4], skptx::f2_pack(e0, e1));
    pk[i] = skptx::pack_bf16x2(e0, e1);
  }
}

// One score row -> P in TMEM columns tP .. tP + 63 (keys 0-63 released on
// bar_lo, keys 64-127 on bar_hi, each after its stores have completed);
// returns the row sum of the fp32 exponentials.  The exponentials of keys
// 64-95 are computed before the wait that releases keys 0-63, so that wait
// finds the first stores already done.
template <bool kPartial>
__device__ __forceinline__ float exp_row_release(const float (&s)[kBlockN], float sl2, float m, int nvalid,
                                                 uint32_t tP, uint32_t bar_lo, uint32_t bar_hi) {
  const uint64_t sl2_2 = skptx::f2_pack(sl2, sl2);
  const uint64_t negm_2 = skptx::f2_pack(-m, -m);
  uint64_t acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = 0;
  uint32_t pa[16], pb[16];
  exp_chunk<kPartial, 0>(s, sl2_2, negm_2, nvalid, pa, acc);
  skptx::tmem_st16(tP, pa);
  exp_chunk<kPartial, 1>(s, sl2_2, negm_2, nvalid, pb, acc);
  skptx::tmem_st16(tP + 16, pb);
  exp_chunk<kPartial, 2>(s, sl2_2, negm_2, nvalid, pa, acc);
  skptx::tmem_wait_st();
  skptx::tc_fence_before();
  skptx::mbar_arrive(bar_lo);
  skptx::tmem_st16(tP + 32, pa);
  exp_chunk<kPartial, 3>(s, sl2_2, negm_2, nvalid, pb, acc);
  skptx::tmem_st16(tP + 48, pb);
  skptx::tmem_wait_st();
  skptx::tc_fence_before();
  skptx::mbar_arrive(bar_hi);
  const uint64_t a = skptx::add2(skptx::add2(acc[0], acc[1]), skptx::add2(acc[2], acc[3]));
  float a0, a1;
  skptx::f2_unpack(a, a0, a1);
  return a0 + a1;
}

// Tiles after the first, scores loaded in two halves: the exponentials of keys
// 0-63 run on the running maximum m while keys 64-127 are still on their way
// from TMEM; the tile's own maximum is checked before anything is released.
// Returns false (nothing released, stores may be in flight) when some row of
// the warp needs m raised by more than 2^kRescaleLog2: s then holds the whole
// masked row for the regular path.  Otherwise the same P and sum as
// exp_row_release with the same m.
template <bool kPartial>
__device__ __forceinline__ bool exp_row_split_load(float (&s)[kBlockN], uint32_t tS, float sl2, float m, int nvalid,
                                                   uint32_t bar_lo, uint32_t bar_hi, float& sum) {
  {
    uint32_t u[2][32];
    skptx::tmem_ld32(tS, u[0]);
    skptx::tmem_ld32(tS + 32, u[1]);
    skptx::tmem_wait_ld();
    skptx::reg_fence(u[0]);
    skptx::reg_fence(u[1]);
#pragma unroll
    for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(u[c / 32][c % 32]);
  }
  uint32_t w[2][32];
  skptx::tmem_ld32(tS + 64, w[0]);  // in flight during the first exponentials
  skptx::tmem_ld32(tS + 96, w[1]);
  if (kPartial) {
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (c >= nvalid) s[c] = -INFINITY;
  }
  const uint64_t sl2_2 = skptx::f2_pack(sl2, sl2);
  const uint64_t negm_2 = skptx::f2_pack(-m, -m);
  uint64_t acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = 0;
  uint32_t pa[16], pb[16];
  exp_chunk<kPartial, 0>(s, sl2_2, negm_2, nvalid, pa, acc);
  skptx::tmem_st16(tS, pa);
  exp_chunk<kPartial, 1>(s, sl2_2, negm_2, nvalid, pb, acc);
  skptx::tmem_st16(tS + 16, pb);
  skptx::tmem_wait_ld();
  skptx::reg_fence(w[0]);
  skptx::reg_fence(w[1]);
#pragma unroll
  for (int c = 64; c < kBlockN; ++c) s[c] = __uint_as_float(w[(c - 64) / 32][c % 32]);
  if (kPartial) {
#pragma unroll
    for (int c = 64; c < kBlockN; ++c)
      if (c >= nvalid) s[c] = -INFINITY;
  }
  const float mt = fmaxf(half_max<0>(s), half_max<64>(s)) * sl2;
  if (__any_sync(0xffffffffu, mt > m + kRescaleLog2)) return false;
  exp_chunk<kPartial, 2>(s, sl2_2, negm_2, nvalid, pa, acc);
  skptx::tmem_wait_st();
  skptx::tc_fence_before();
  skptx::mbar_arrive(bar_lo);
  skptx::tmem_st16(tS + 32, pa);
  exp_chunk<kPartial, 3>(s, sl2_2, negm_2, nvalid, pb, acc);
  skptx::tmem_st16(tS + 48, pb);
  skptx::tmem_wait_st();
  skptx::tc_fence_before();
  skptx::mbar_arrive(bar_hi);
  const uint64_t a = skptx::add2(skptx::add2(acc[0], acc[1]), skptx::add2(acc[2], acc[3]));
  float a0, a1;
  skptx::f2_unpack(a, a0, a1);
  sum = a0 + a1;
  return true;
}


// S = Q K^T: 128 x 128 x D, both operands K-major in shared memory
// (64-column sub-tiles kSub bytes apart).  Warp-collective.
template <int D>
__device__ __forceinline__ void issue_s_p(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc) {
  using L = PSmemLayout<D>;
  constexpr uint32_t idS = skptx::idesc_bf16_f32(kBlockM, kBlockN, false);
  skptx::mma_ss_block<D / 16, (L::kSub >> 4)>(d_tmem, q_desc, k_desc, idS, 0u);
}

// O += P V: P (128 x 128 bf16) from TMEM, 8 columns per 16 keys; V (MN-major,
// head_dim contiguous, 128-byte swizzle) from shared memory, 2048 B per 16
// keys.  ksteps < 8: only the first 16 * ksteps keys (the rest of the tile is
// past the valid keys and P is zero there).  Warp-collective.
template <int D>
__device__ __forceinline__ void issue_pv_p(uint32_t o_tmem, uint32_t p_tmem, uint64_t v_desc, bool accumulate,
                                           int ksteps = kBlockN / 16) {
  constexpr uint32_t idO = skptx::idesc_bf16_f32(kBlockM, D, true);
  skptx::mma_ts_block<(2048 >> 4)>(o_tmem, p_tmem, v_desc, idO, accumulate ? 1u : 0u, ksteps);
}

// Zero V rows [r0, r1) of a stage (every 64-column sub-tile; a row's 128 bytes
// stay together under the swizzle) and make the zeros visible to the tensor
// core.  Warp-collective.
template <int D>
__device__ __forceinline__ void zero_v_rows(uint32_t vbase, int r0, int r1, int lane) {
  constexpr int kChunks = (D / 64) * 8;  // 16-byte chunks per row
  const int n = (r1 - r0) * kChunks;
  for (int i = lane; i < n; i += 32) {
    const int r = r0 + i / kChunks;
    const int rem = i % kChunks;
    skptx::st_shared_v4(vbase + (rem / 8) * (kBlockM * 128u) + static_cast<uint32_t>(r) * 128u + (rem % 8) * 16u,
                        0u, 0u, 0u, 0u);
  }
  skptx::fence_proxy_async_smem();
  __syncwarp();
}

// The kernel's shared context: shared-memory base, TMEM base, the bounded
// waiter and the barrier array (index -> shared address).
template <int D>
struct PCtx {
  using L = PSmemLayout<D>;
  uint32_t sbase;
  uint32_t tmem;
  Waiter W;
  __device__ __forceinline__ uint32_t bar(int i) const { return sbase + L::kBar + 8u * static_cast<uint32_t>(i); }
};

// ---------------------------------------------------------------- TMA producer
// Q tiles per unit, K and V tiles into rings, in the order the MMAs need them.
template <int D, typename Params>
__device__ __forceinline__ void tma_producer(const Params& p, const PCtx<D>& cx, int lane) {
  using L = PSmemLayout<D>;
  constexpr bool kShared = std::is_same<Params, VarlenParams>::value;
  constexpr int KS = L::kKS;
  constexpr int VS = L::kVS;
  const uint32_t sbase = cx.sbase;
  const Waiter& W = cx.W;
  auto bar = [&](int i) { return cx.bar(i); };
  const int n_units = p.n_units;
  int kq = 0, vq = 0;    // K / V loads issued (ring positions)
  int qn[2] = {0, 0};    // Q loads issued per tile
  int prev_bl = -1;
  bool ok = true;
  for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
    const PUnit t = decode_unit(p, u);
    if (!t.compute) continue;
    const int hkv = t.hq / p.group;
    if (t.bl != prev_bl && !(kShared && prev_bl >= 0)) {
      if (lane == 0) {
        skptx::prefetch_tmap(q_map(p, t));
        if (t.nkp > 0) { skptx::prefetch_tmap(k_map(p, t, true)); skptx::prefetch_tmap(v_map(p, t, true)); }
        if (t.nks > 0) { skptx::prefetch_tmap(k_map(p, t, false)); skptx::prefetch_tmap(v_map(p, t, false)); }
      }
      __syncwarp();
    }
    prev_bl = t.bl;
    for (int x = 0; x < 2 && ok; ++x) {
      if (qn[x] > 0 && !W.wait_warp(bar(L::bQEmpty + x), (qn[x] - 1) & 1)) { ok = false; break; }
      skptx::mbar_arrive_expect_tx_elect(bar(L::bQFull + x), L::kQTile);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        skptx::tma_load_3d_elect(sbase + L::kQ + x * L::kQTile + c * L::kSub, q_map(p, t),
                                 bar(L::bQFull + x), c * 64, t.hq, t.q_off + t.row0 + x * kBlockM);
      ++qn[x];
    }
    // K(j) and V(j) in the order the MMAs need them.
    for (int j = 0; ok && j < t.n_tiles; ++j) {
      const bool pre = j < t.tP;
      const int key0 = t.k_off + (pre ? j : j - t.tP) * kBlockN;
      {
        const int s = kq % KS;
        if (kq >= KS && !W.wait_warp(bar(L::bKEmpty + s), ((kq / KS) - 1) & 1)) { ok = false; break; }
        const CUtensorMap* mk = k_map(p, t, pre);
        skptx::mbar_arrive_expect_tx_elect(bar(L::bKFull + s), L::kKVTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          skptx::tma_load_3d_elect(sbase + L::kK + s * L::kKVTile + c * L::kSub, mk, bar(L::bKFull + s),
                                   c * 64, hkv, key0);
        ++kq;
      }
      {
        const int s = vq % VS;
        if (vq >= VS && !W.wait_warp(bar(L::bVEmpty + s), ((vq / VS) - 1) & 1)) { ok = false; break; }
        const CUtensorMap* mv = v_map(p, t, pre);
        skptx::mbar_arrive_expect_tx_elect(bar(L::bVFull + s), L::kKVTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          skptx::tma_load_3d_elect(sbase + L::kV + s * L::kKVTile + c * L::kSub, mv, bar(L::bVFull + s),
                                   c * 64, hkv, key0);
        ++vq;
      }
    }
  }
  // Drain: no copy issued by this CTA may still be landing when it exits.
  // Only the last ring's worth of loads can be outstanding (an earlier load's
  // stage was reused, so it had landed); on the normal path all have landed.
  for (int x = 0; x < 2; ++x)
    if (qn[x] > 0) W.drain_warp(bar(L::bQFull + x), (qn[x] - 1) & 1);
  for (int i = (kq > KS ? kq - KS : 0); i < kq; ++i) W.drain_warp(bar(L::bKFull + i % KS), (i / KS) & 1);
  for (int i = (vq > VS ? vq - VS : 0); i < vq; ++i) W.drain_warp(bar(L::bVFull + i % VS), (i / VS) & 1);
}

// ---------------------------------------------------------------- MMA issuer
// Per KV tile j: PV_A(j) (in two halves as P_A(j) is released), S_A(j+1),
// PV_B(j), S_B(j+1).
template <int D, typename Params>
__device__ __forceinline__ void mma_issuer(const Params& p, const PCtx<D>& cx, int lane) {
  using L = PSmemLayout<D>;
  constexpr bool kShared = std::is_same<Params, VarlenParams>::value;
  constexpr int KS = L::kKS;
  constexpr int VS = L::kVS;
  const uint32_t sbase = cx.sbase;
  const uint32_t tmem = cx.tmem;
  const Waiter& W = cx.W;
  auto bar = [&](int i) { return cx.bar(i); };
  const int n_units = p.n_units;
  const uint64_t dQ = skptx::sdesc_sw128(sbase + L::kQ, 16, 1024);
  const uint64_t dK = skptx::sdesc_sw128(sbase + L::kK, 16, 1024);
  const uint64_t dV = skptx::sdesc_sw128(sbase + L::kV, L::kSub, 1024);
  const uint32_t tS[2] = {tmem, tmem + 128u};
  const uint32_t tO[2] = {tmem + 256u, tmem + 384u};
  bool ok = true;
  // Test hook for the bounded-wait path: MmaDone is only committed after the
  // loop, so this wait runs out and every role aborts.
  if (p.test_stall) ok = W.wait_warp(bar(L::bMmaDone), 0);
  int kc = 0, vc = 0;       // K / V ring positions consumed
  int un = 0;               // computed units so far (Q / O phases)
  int pc[2] = {0, 0};       // P tiles consumed per tile (PFull phases)
  auto wait_k = [&]() -> bool {
    return W.wait_warp(bar(L::bKFull + kc % KS), (kc / KS) & 1);
  };
  for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
    const PUnit t = decode_unit(p, u);
    if (!t.compute) continue;
    const int n = t.n_tiles;
    if (!W.wait_warp(bar(L::bQFull + 0), un & 1) || !W.wait_warp(bar(L::bQFull + 1), un & 1) || !wait_k()) {
      ok = false;
      break;
    }
    skptx::tc_fence_after();
    const uint64_t dKs = dK + (((kc % KS) * L::kKVTile) >> 4);
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      issue_s_p<D>(tS[x], dQ + ((x * L::kQTile) >> 4), dKs);
      skptx::mma_commit_elect(bar(L::bSFull + x));
      if (n == 1) skptx::mma_commit_elect(bar(L::bQEmpty + x));
    }
    skptx::mma_commit_elect(bar(L::bKEmpty + kc % KS));
    ++kc;
    for (int j = 0; j < n; ++j) {
      const int vs = vc % VS;
      const uint64_t dVs = dV + ((vs * L::kKVTile) >> 4);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const uint64_t dQx = dQ + ((x * L::kQTile) >> 4);
        // P arrives in two halves (keys 0-63, then 64-127): the first half
        // of PV runs while the softmax still exponentiates the second.
        if (!W.wait_warp(bar(L::bPLo + x), pc[x] & 1)) { ok = false; break; }
        if (x == 0 && !W.wait_warp(bar(L::bVFull + vs), (vc / VS) & 1)) { ok = false; break; }
        int ksteps = kBlockN / 16;
        if (kShared) {
          const int nv = tile_valid(j, t.tP, t.nkp, t.nks);
          ksteps = (nv + 15) / 16;
          if (x == 0 && nv < ksteps * 16) zero_v_rows<D>(sbase + L::kV + vs * L::kKVTile, nv, ksteps * 16, lane);
        }
        skptx::tc_fence_after();
        issue_pv_p<D>(tO[x], tS[x], dVs, j > 0, ksteps < 4 ? ksteps : 4);
        if (!W.wait_warp(bar(L::bPHi + x), pc[x] & 1)) { ok = false; break; }
        ++pc[x];
        if (ksteps > 4) {
          skptx::tc_fence_after();
          issue_pv_p<D>(tO[x], tS[x] + 32u, dVs + ((4 * 2048) >> 4), true, ksteps - 4);
        }
        if (x == 1) {
          skptx::mma_commit_elect(bar(L::bVEmpty + vs));
          ++vc;
        }
        if (j == n - 1) skptx::mma_commit_elect(bar(L::bOFull + x));
        if (j + 1 < n) {
          if (x == 0 && !wait_k()) { ok = false; break; }
          skptx::tc_fence_after();
          issue_s_p<D>(tS[x], dQx, dK + (((kc % KS) * L::kKVTile) >> 4));
          skptx::mma_commit_elect(bar(L::bSFull + x));
          if (j + 1 == n - 1) skptx::mma_commit_elect(bar(L::bQEmpty + x));
          if (x == 1) {
            skptx::mma_commit_elect(bar(L::bKEmpty + kc % KS));
            ++kc;
          }
        }
      }
      if (!ok) break;
    }
    ++un;
  }
  // Every MMA this warp issued has finished before TMEM is released.
  skptx::mma_commit_elect(bar(L::bMmaDone));
  W.drain_warp(bar(L::bMmaDone), 0);
}

// ---------------------------------------------------------------- softmax, one thread per row
// Warps 0-3 tile A, 4-7 tile B: thread t of a warpgroup owns query row t of
// its tile (TMEM lane t) and all 128 columns of its score row.
template <int D, bool kScatter, typename Params>
__device__ __forceinline__ void softmax_rows(const Params& p, const PCtx<D>& cx, int warp) {
  using L = PSmemLayout<D>;
  const uint32_t tmem = cx.tmem;
  const Waiter& W = cx.W;
  auto bar = [&](int i) { return cx.bar(i); };
  const int n_units = p.n_units;
  const int x = warp / 4;            // query tile of this warpgroup
  const int r = threadIdx.x % 128;   // row in tile == TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
  const uint32_t tS_ = tmem + lane_base + static_cast<uint32_t>(x) * 128;
  const uint32_t tO = tmem + lane_base + 256 + static_cast<uint32_t>(x) * 128;
  const float sl2 = p.scale_log2;
  int sc = 0;  // score tiles consumed (SFull phases)
  int un = 0;  // computed units so far (OFull phases)
  bool ok = true;
  for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
    const PUnit t = decode_unit(p, u);
    const int row = t.row0 + x * kBlockM + r;
    if (!t.compute) {
      if (row < t.sq) {
        uint4* dst = reinterpret_cast<uint4*>(unit_row_ptr<kScatter>(p, t, row));
#pragma unroll
        for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0, 0, 0, 0);
      }
      continue;
    }
    float m_run = 0.f;  // running (possibly stale) max of scale*log2(e)*s
    float l_run = 0.f;  // running sum of exponentials
    for (int j = 0; j < t.n_tiles; ++j) {
      ok = W.wait_warp(bar(L::bSFull + x), sc & 1);
      if (!ok) break;
      ++sc;
      skptx::tc_fence_after();
      const int nvalid = tile_valid(j, t.tP, t.nkp, t.nks);
      const bool partial = nvalid < kBlockN;
      float s[kBlockN];
      if (j > 0) {  // the common case: exponentials start on the running max
        float sum;
        const bool done =
            partial ? exp_row_split_load<true>(s, tS_, sl2, m_run, nvalid, bar(L::bPLo + x), bar(L::bPHi + x), sum)
                    : exp_row_split_load<false>(s, tS_, sl2, m_run, nvalid, bar(L::bPLo + x), bar(L::bPHi + x), sum);
        if (done) {
          l_run += sum;
          continue;
        }
        skptx::tmem_wait_st();  // the early P stores land before they are overwritten
      } else {  // first tile of the unit: its maximum starts the running max
        uint32_t uu[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) skptx::tmem_ld32(tS_ + c * 32, uu[c]);
        skptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) skptx::reg_fence(uu[c]);
#pragma unroll
        for (int c = 0; c < kBlockN; ++c) s[c] = __uint_as_float(uu[c / 32][c % 32]);
      }
      if (partial && j == 0) {
#pragma unroll
        for (int c = 0; c < kBlockN; ++c)
          if (c >= nvalid) s[c] = -INFINITY;
      }
      const float m_tile = fmaxf(half_max<0>(s), half_max<64>(s)) * sl2;
      float alpha = 1.f;
      bool raise = false;
      if (j == 0) {
        m_run = m_tile;
      } else if (m_tile > m_run + kRescaleLog2) {
        alpha = skptx::ex2_approx(m_run - m_tile);
        m_run = m_tile;
        raise = true;
      }
      // O_X holds the sum over tiles < j (PV_X(j-1) finished before S_X(j)
      // was complete); rescale it before PV_X(j) accumulates (rare: only
      // when the row maximum grows by more than 2^kRescaleLog2).
      if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          skptx::tmem_ld32(tO + c * 32, o);
          skptx::tmem_wait_ld();
          skptx::reg_fence(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          skptx::tmem_st32(tO + c * 32, o);
        }
      }
      const float sum = partial ? exp_row_release<true>(s, sl2, m_run, nvalid, tS_, bar(L::bPLo + x), bar(L::bPHi + x))
                                : exp_row_release<false>(s, sl2, m_run, nvalid, tS_, bar(L::bPLo + x), bar(L::bPHi + x));
      l_run = l_run * alpha + sum;
    }
    if (!ok) break;
    // ---------------------------------------------------------- epilogue
    ok = W.wait_warp(bar(L::bOFull + x), un & 1);
    if (!ok) break;
    ++un;
    skptx::tc_fence_after();
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    uint16_t* orow = unit_row_ptr<kScatter>(p, t, row < t.sq ? row : 0);
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      skptx::tmem_ld32(tO + c * 32, o);
      skptx::tmem_wait_ld();
      skptx::reg_fence(o);
      if (row < t.sq) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
        if (row < t.qv) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = skptx::pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
            w.y = skptx::pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
            w.z = skptx::pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
            w.w = skptx::pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
            dst[v] = w;
          }
        } else {
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(0, 0, 0, 0);
        }
      }
    }
    // O_X has been read into registers: the next unit's PV_X(0) may
    // overwrite it (ordered by this thread's later PFull arrive).
    skptx::tc_fence_before();
  }
}

// ---------------------------------------------------------------- the kernel
// Params: AttnParams (batch rows, split K/V) or VarlenParams (packed segments).
template <int D, bool kScatter, typename Params>
__global__ void __launch_bounds__(kPThreads, 1) attn_fwd_persistent_kernel(const __grid_constant__ Params p) {
  using L = PSmemLayout<D>;
  constexpr int KS = L::kKS;
  constexpr int VS = L::kVS;
  constexpr int kTma = 8;
  constexpr int kMma = 9;
  constexpr int kSoftWarps = 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = skptx::smem_addr(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      skptx::mbar_init(bar(L::bQFull + x), 1);
      skptx::mbar_init(bar(L::bQEmpty + x), 1);
      skptx::mbar_init(bar(L::bSFull + x), 1);
      skptx::mbar_init(bar(L::bPLo + x), kBlockM);
      skptx::mbar_init(bar(L::bPHi + x), kBlockM);
      skptx::mbar_init(bar(L::bOFull + x), 1);
    }
    for (int s = 0; s < KS; ++s) {
      skptx::mbar_init(bar(L::bKFull + s), 1);
      skptx::mbar_init(bar(L::bKEmpty + s), 1);
    }
    for (int s = 0; s < VS; ++s) {
      skptx::mbar_init(bar(L::bVFull + s), 1);
      skptx::mbar_init(bar(L::bVEmpty + s), 1);
    }
    skptx::mbar_init(bar(L::bMmaDone), 1);
    *abort_flag = 0;
    skptx::fence_mbarrier_init();
  }
  if (warp == kMma) {
    skptx::tmem_alloc(skptx::smem_addr(tmem_slot), kTmemCols);
    skptx::tmem_relinquish();
  }
  skptx::tc_fence_before();
  __syncthreads();
  skptx::tc_fence_after();
  const PCtx<D> cx{sbase, *tmem_slot, Waiter{abort_flag, p.status, p.wait_limit_ns}};
  // Each role sets its register budget at the top of its own branch (the
  // compiler allocates every branch within the budget it sets).
  if (warp >= kSoftWarps) {
    skptx::setmaxnreg_dec<kOtherRegs>();
    if (warp == kTma) tma_producer<D>(p, cx, lane);
    else if (warp == kMma) mma_issuer<D>(p, cx, lane);
  } else {
    skptx::setmaxnreg_inc<kSoftmaxRegs>();
    softmax_rows<D, kScatter>(p, cx, warp);
  }

  skptx::tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
    skptx::tc_fence_after();
    skptx::tmem_dealloc(cx.tmem, kTmemCols);
  }
}

}  // namespace skattn
