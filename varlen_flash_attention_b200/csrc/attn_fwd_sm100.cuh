// Split-KV tail-padded attention forward for sm_100a.
//
// One CTA computes one 128-row query tile of one (batch row, query head):
//   O = softmax(scale * Q K*^T) V*,  K*/V* = cat(prefix, suffix)[0:real_len]
// ("sglang PR 26973", forward_with_replicated_kv_prefix; "sglang PR 30107",
// tail_attn_meta / tail-pad layout invariant).  The concatenation is never
// built: the KV tile loop first walks the prefix tensor map, then the suffix
// tensor map.  Each map's sequence extent is clipped on the host to the valid
// keys of this batch row, so TMA never fetches a pad byte (out-of-range rows
// arrive as zeros) and tiles past real_len are never issued; the one partial
// tile of each source is masked column-wise in the softmax.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t of the tile (TMEM lane t);
//              online softmax in fp32 (exp2 with scale*log2(e) folded in),
//              P written back to TMEM as bf16, O rescaled in TMEM, epilogue.
//   warp 4     TMA producer: Q once, then K/V tiles into a 2-stage ring.
//   warp 5     TMEM allocator + single-thread tcgen05.mma issuer:
//              S_j = Q K_j^T (SS, both K-major) into one of two S buffers,
//              O += P_{j-1} V_{j-1} (A = P from TMEM, B = V MN-major).
// TMEM (512 columns): S0 [0,128), S1 [128,256), O [256, 256+D).
// Every wait is bounded (globaltimer); on expiry the CTA raises a device
// status word, drains its own copies, frees TMEM and exits.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace skattn {

constexpr int kBlockM = 128;    // query rows per tile
constexpr int kBlockN = 128;    // keys per KV tile
constexpr int kMaxBatch = 8;    // batch rows per launch (tensor maps live in parameter space)
constexpr int kThreads = 192;
constexpr int kStages = 2;      // K/V smem ring depth
constexpr uint32_t kTmemCols = 512;
constexpr int32_t kStatusTimeout = 4;

struct alignas(64) AttnParams {
  CUtensorMap tm_q[kMaxBatch];
  CUtensorMap tm_kp[kMaxBatch];
  CUtensorMap tm_vp[kMaxBatch];
  CUtensorMap tm_ks[kMaxBatch];
  CUtensorMap tm_vs[kMaxBatch];
  int32_t q_valid[kMaxBatch];   // query rows that are real
  int32_t n_prefix[kMaxBatch];  // valid prefix keys = min(Sp, real_len)
  int32_t n_suffix[kMaxBatch];  // valid suffix keys = max(0, real_len - Sp)
  uint16_t* out;                // element (b0, 0, 0, 0) of this launch's first batch row
  int64_t out_sb, out_ss, out_sh;
  int32_t Sq;
  int32_t group;                // num_q_heads / num_kv_heads
  float scale_log2;             // softmax_scale * log2(e)
  int32_t* status;              // device status word
  uint64_t wait_limit_ns;
};

template <int D>
struct SmemLayout {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr uint32_t kSub = kBlockM * 128;          // one 64-column (128 B) swizzled sub-tile
  static constexpr uint32_t kQBytes = kBlockM * D * 2;
  static constexpr uint32_t kKVBytes = kBlockN * D * 2;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kQBytes;
  static constexpr uint32_t kV = kK + kStages * kKVBytes;
  static constexpr uint32_t kBar = kV + kStages * kKVBytes;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bKFull = 1;                   // + stage
  static constexpr int bVFull = bKFull + kStages;    // + stage
  static constexpr int bKVEmpty = bVFull + kStages;  // + stage
  static constexpr int bSFull = bKVEmpty + kStages;  // + buffer (2)
  static constexpr int bPFull = bSFull + 2;          // + buffer (2)
  static constexpr int bOReady = bPFull + 2;
  static constexpr int bMmaDone = bOReady + 1;
  static constexpr int kNumBars = bMmaDone + 1;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kEnd = kMisc + 16;
  // +1024 slack to align the dynamic base; at least ~116 KB so one CTA per SM
  // (the CTA allocates all 512 TMEM columns).
  static constexpr uint32_t kAlloc = (kEnd + 1024) > 120 * 1024 ? (kEnd + 1024) : 120 * 1024;
};

// Bounded mbarrier wait shared by all roles.  Returns false on timeout or when
// another thread of the CTA already aborted.
struct Waiter {
  volatile int* abort_flag;
  int32_t* status;
  uint64_t limit_ns;

  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
    if (skptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = skptx::globaltimer_ns();
    uint32_t it = 0;
    while (true) {
      if (skptx::mbar_try_wait(bar, parity)) return true;
      if ((++it & 63u) == 0) {
        if (*abort_flag) return false;
        if (skptx::globaltimer_ns() - t0 > limit_ns) {
          *abort_flag = 1;
          atomicOr(status, kStatusTimeout);
          return false;
        }
      }
    }
  }
};

__device__ __forceinline__ void store_zero_rows(uint16_t* base, int64_t ss, int r_begin,
                                                int r_end, int D, int tid, int nthreads) {
  const int chunks = D / 8;  // 16-byte chunks per row
  const int total = (r_end - r_begin) * chunks;
  for (int idx = tid; idx < total; idx += nthreads) {
    const int r = r_begin + idx / chunks;
    const int c = idx % chunks;
    *reinterpret_cast<uint4*>(base + static_cast<int64_t>(r) * ss + c * 8) = make_uint4(0, 0, 0, 0);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using L = SmemLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = skptx::smem_addr(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  const int q_tile = blockIdx.x;
  const int hq = blockIdx.y;
  const int bl = blockIdx.z;
  const int row0 = q_tile * kBlockM;
  const int qv = p.q_valid[bl];
  const int nkp = p.n_prefix[bl];
  const int nks = p.n_suffix[bl];
  const int tP = (nkp + kBlockN - 1) / kBlockN;
  const int tS = (nks + kBlockN - 1) / kBlockN;
  const int n_tiles = tP + tS;
  uint16_t* out_bh = p.out + static_cast<int64_t>(bl) * p.out_sb + static_cast<int64_t>(hq) * p.out_sh;

  if (row0 >= qv || n_tiles == 0) {
    // The whole tile is pad rows, or this batch row has no valid key: exact zeros.
    const int r_end = min(row0 + kBlockM, p.Sq);
    store_zero_rows(out_bh, p.out_ss, row0, r_end, D, threadIdx.x, kThreads);
    return;
  }

  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  if (threadIdx.x == 0) {
    skptx::mbar_init(bar(L::bQFull), 1);
    for (int s = 0; s < kStages; ++s) {
      skptx::mbar_init(bar(L::bKFull + s), 1);
      skptx::mbar_init(bar(L::bVFull + s), 1);
      skptx::mbar_init(bar(L::bKVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      skptx::mbar_init(bar(L::bSFull + b), 1);
      skptx::mbar_init(bar(L::bPFull + b), kBlockM);
    }
    skptx::mbar_init(bar(L::bOReady), 1);
    skptx::mbar_init(bar(L::bMmaDone), 1);
    *abort_flag = 0;
    skptx::fence_mbarrier_init();
  }
  if (warp == 5) {
    skptx::tmem_alloc(skptx::smem_addr(tmem_slot), kTmemCols);
    skptx::tmem_relinquish();
  }
  skptx::tc_fence_before();
  __syncthreads();
  skptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, p.status, p.wait_limit_ns};

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int hkv = hq / p.group;
      skptx::prefetch_tmap(&p.tm_q[bl]);
      if (tP > 0) { skptx::prefetch_tmap(&p.tm_kp[bl]); skptx::prefetch_tmap(&p.tm_vp[bl]); }
      if (tS > 0) { skptx::prefetch_tmap(&p.tm_ks[bl]); skptx::prefetch_tmap(&p.tm_vs[bl]); }
      skptx::mbar_arrive_expect_tx(bar(L::bQFull), L::kQBytes);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        skptx::tma_load_3d(sbase + L::kQ + c * L::kSub, &p.tm_q[bl], bar(L::bQFull), c * 64, hq, row0);
      int j = 0;
      for (; j < n_tiles; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !W.wait(bar(L::bKVEmpty + s), ((j / kStages) - 1) & 1)) break;
        const bool pre = j < tP;
        const CUtensorMap* mk = pre ? &p.tm_kp[bl] : &p.tm_ks[bl];
        const CUtensorMap* mv = pre ? &p.tm_vp[bl] : &p.tm_vs[bl];
        const int key0 = (pre ? j : j - tP) * kBlockN;
        const uint32_t k_dst = sbase + L::kK + s * L::kKVBytes;
        const uint32_t v_dst = sbase + L::kV + s * L::kKVBytes;
        skptx::mbar_arrive_expect_tx(bar(L::bKFull + s), L::kKVBytes);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          skptx::tma_load_3d(k_dst + c * L::kSub, mk, bar(L::bKFull + s), c * 64, hkv, key0);
        skptx::mbar_arrive_expect_tx(bar(L::bVFull + s), L::kKVBytes);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          skptx::tma_load_3d(v_dst + c * L::kSub, mv, bar(L::bVFull + s), c * 64, hkv, key0);
      }
      // Drain: no copy issued by this CTA may still be landing when it exits.
      // On the normal path every wait below has already completed.
      const Waiter drain{abort_flag, p.status, p.wait_limit_ns};
      drain.wait(bar(L::bQFull), 0);
      for (int jj = (j > kStages ? j - kStages : 0); jj < j; ++jj) {
        const int s = jj % kStages;
        drain.wait(bar(L::bKFull + s), (jj / kStages) & 1);
        drain.wait(bar(L::bVFull + s), (jj / kStages) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = skptx::idesc_bf16_f32(kBlockM, kBlockN, false);
      constexpr uint32_t idO = skptx::idesc_bf16_f32(kBlockM, D, true);
      const uint32_t sQ = sbase + L::kQ;
      const uint32_t tO = tmem + 256;
      bool ok = W.wait(bar(L::bQFull), 0);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j % kStages;
          if (!W.wait(bar(L::bKFull + s), (j / kStages) & 1)) { ok = false; break; }
          // S_j overwrites the buffer that held P_{j-2}: PV_{j-2} must have finished.
          if (j >= 2 && !W.wait(bar(L::bOReady), (j - 2) & 1)) { ok = false; break; }
          skptx::tc_fence_after();
          const uint32_t sK = sbase + L::kK + s * L::kKVBytes;
          const uint32_t dS = tmem + static_cast<uint32_t>(j & 1) * 128;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k / 4) * L::kSub + (k % 4) * 32;
            skptx::mma_ss(dS, skptx::sdesc_sw128(sQ + off, 16, 1024),
                          skptx::sdesc_sw128(sK + off, 16, 1024), idS, k > 0 ? 1u : 0u);
          }
          skptx::mma_commit(bar(L::bSFull + (j & 1)));
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int s = jj % kStages;
          const int b = jj & 1;
          if (!W.wait(bar(L::bPFull + b), (jj >> 1) & 1)) { ok = false; break; }
          if (!W.wait(bar(L::bVFull + s), (jj / kStages) & 1)) { ok = false; break; }
          skptx::tc_fence_after();
          const uint32_t sV = sbase + L::kV + s * L::kKVBytes;
          const uint32_t tP_ = tmem + static_cast<uint32_t>(b) * 128;
#pragma unroll
          for (int k = 0; k < kBlockN / 16; ++k) {
            skptx::mma_ts(tO, tP_ + k * 8, skptx::sdesc_sw128(sV + k * 2048, L::kSub, 1024), idO,
                          (jj > 0 || k > 0) ? 1u : 0u);
          }
          skptx::mma_commit(bar(L::bKVEmpty + s));
          skptx::mma_commit(bar(L::bOReady));
        }
      }
      // Every MMA this thread issued has finished before TMEM is released.
      skptx::mma_commit(bar(L::bMmaDone));
      const Waiter drain{abort_flag, p.status, p.wait_limit_ns};
      drain.wait(bar(L::bMmaDone), 0);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int r = threadIdx.x;  // row in tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;  // running max of scale*log2(e)*s
    float l_run = 0.f;        // running sum of exponentials
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int b = j & 1;
      ok = __all_sync(0xffffffffu, W.wait(bar(L::bSFull + b), (j >> 1) & 1));
      if (!ok) break;
      skptx::tc_fence_after();
      const uint32_t tS_ = tmem + lane_base + static_cast<uint32_t>(b) * 128;
      uint32_t u[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) skptx::tmem_ld32(tS_ + c * 32, u[c]);
      skptx::tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) skptx::reg_fence(u[c]);

      const int nvalid = (j < tP) ? min(kBlockN, nkp - j * kBlockN) : min(kBlockN, nks - (j - tP) * kBlockN);
      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(u[c / 32][c % 32]);
      if (nvalid < kBlockN) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= nvalid) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
      const float m_new = fmaxf(m_run, mx * sl2);
      const float alpha = skptx::ex2_approx(m_run - m_new);
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = skptx::ex2_approx(fmaf(s[c], sl2, -m_new));
      if (nvalid < kBlockN) {
        // exact zeros for masked columns (also when scale == 0, where -inf * 0 is NaN)
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= nvalid) s[c] = 0.f;
      }
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) sum += s[c];
      l_run = l_run * alpha + sum;
      m_run = m_new;
      // P (bf16 pairs) overwrites the first 64 columns of this S buffer.
      uint32_t pk[2][32];
#pragma unroll
      for (int i = 0; i < 64; ++i) pk[i / 32][i % 32] = skptx::pack_bf16x2(s[2 * i], s[2 * i + 1]);
      skptx::tmem_st32(tS_, pk[0]);
      skptx::tmem_st32(tS_ + 32, pk[1]);

      if (j > 0) {
        // O holds sum over tiles < j; rescale once PV_{j-1} has landed.
        ok = __all_sync(0xffffffffu, W.wait(bar(L::bOReady), (j - 1) & 1));
        if (!ok) break;
        skptx::tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          const uint32_t tO = tmem + lane_base + 256;
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
      }
      skptx::tmem_wait_st();
      skptx::tc_fence_before();
      skptx::mbar_arrive(bar(L::bPFull + b));
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = __all_sync(0xffffffffu, W.wait(bar(L::bOReady), (n_tiles - 1) & 1));
    if (ok) {
      skptx::tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      const int row = row0 + r;
      uint16_t* orow = out_bh + static_cast<int64_t>(row) * p.out_ss;
      const uint32_t tO = tmem + lane_base + 256;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        skptx::tmem_ld32(tO + c * 32, o);
        skptx::tmem_wait_ld();
        skptx::reg_fence(o);
        if (row < p.Sq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
          if (row < qv) {
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
    }
  }

  skptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    skptx::tc_fence_after();
    skptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace skattn
