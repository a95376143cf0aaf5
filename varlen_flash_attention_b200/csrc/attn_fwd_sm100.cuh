// Split-KV tail-padded attention forward for sm_100a.
//
// One CTA computes two 128-row query tiles (A and B, 256 consecutive rows) of
// one (entry, query head), an entry being a batch row or, for packed varlen
// input, one segment:
//   O = softmax(scale * Q K*^T) V*,  K*/V* = cat(prefix, suffix)[0:real_len]
// ("sglang PR 26973", forward_with_replicated_kv_prefix; "sglang PR 30107",
// tail_attn_meta / tail-pad layout invariant).  The concatenation is never
// built: the KV tile loop first walks the prefix tensor map, then the suffix
// tensor map.  Each map's sequence extent is clipped on the host to the valid
// keys of this batch row, so TMA never fetches a pad byte (rows past the
// extent arrive as zeros) and tiles past real_len are never issued; the one
// partial tile of each source is masked column-wise in the softmax.
//
// Warp roles (320 threads):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread t of a
//              warpgroup owns query row t of its tile (TMEM lane t).  Online
//              softmax in fp32 with exp2 (scale*log2 e folded in); the running
//              max is only raised when a tile's max exceeds it by more than
//              kRescaleLog2 (then O and l are rescaled), so most tiles skip the
//              O round trip through registers.  P (bf16) goes to shared memory
//              in the 128-byte-swizzled K-major layout the PV MMA reads.
//   warp 8     TMA producer: both Q tiles once, then K and V tiles into rings.
//   warp 9     TMEM allocator + tcgen05.mma issuer.
// Because P does not live in the S columns, S_X(j+1) is issued as soon as the
// softmax of tile X has read S_X(j) into registers: the next scores are ready
// when the softmax finishes, so each tile's critical path is its softmax alone
// and the two tiles' softmaxes and all MMAs overlap.  The issuer polls the
// four op streams (S_A, S_B, PV_A, PV_B) and issues whichever is ready.
// With head_dim 128 the two tiles share one P buffer (shared memory is full):
// softmax B(j) stores P after PV_A(j) has read it, softmax A(j+1) after
// PV_B(j), which keeps the two tiles half a step apart.
// Warps 8 and 9 run their loops warp-convergently (operands stay warp-uniform)
// and let one elected lane issue each TMA / MMA / commit; a divergent
// single-lane issuer feeds the tensor pipe measurably slower.
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+D), O_B [384,384+D).
// Every wait is bounded (globaltimer); on expiry the CTA raises a device
// status word, drains its own copies, frees TMEM and exits.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace skattn {

constexpr int kBlockM = 128;     // query rows per tile
constexpr int kTilesPerCta = 2;  // query tiles per CTA
constexpr int kRowsPerCta = kBlockM * kTilesPerCta;
constexpr int kBlockN = 128;     // keys per KV tile
constexpr int kMaxBatch = 8;     // batch rows per launch (tensor maps live in parameter space)
constexpr int kMaxOutDst = 8;    // destinations of a scattered output (ranks of one node)
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kKStages = 2;      // K smem ring depth
constexpr int kVStages = 2;      // V smem ring depth
constexpr uint32_t kTmemCols = 512;
constexpr int32_t kStatusTimeout = 4;
constexpr float kRescaleLog2 = 8.0f;  // keep a stale max while the new one is within 2^8

struct alignas(64) AttnParams {
  CUtensorMap tm_q[kMaxBatch];
  CUtensorMap tm_kp[kMaxBatch];
  CUtensorMap tm_vp[kMaxBatch];
  CUtensorMap tm_ks[kMaxBatch];
  CUtensorMap tm_vs[kMaxBatch];
  int32_t q_valid[kMaxBatch];   // query rows that are real
  int32_t n_prefix[kMaxBatch];  // valid prefix keys = min(Sp, real_len)
  int32_t n_suffix[kMaxBatch];  // valid suffix keys = max(0, real_len - Sp)
  int32_t sq[kMaxBatch];        // output rows of the entry (rows in [q_valid, sq) are written as zeros)
  int64_t out_off[kMaxBatch];   // element offset of the entry's row 0, head 0 from `out` (or a destination)
  uint16_t* out;
  int64_t out_ss, out_sh;
  // Scattered output (out_chunk > 0): row s goes to out_dst[s / out_chunk] at
  // row s % out_chunk, e.g. the receive buffers of the ranks that own each
  // sequence chunk (the output all-to-all of the Ulysses form).  The pointers
  // may address peer GPUs' memory; only plain stores are issued to them, and
  // they are performed by the time the kernel completes (no per-CTA fence: a
  // CTA exits while its stores drain, and the caller's barrier after the
  // kernel publishes them).
  int32_t out_chunk;
  uint16_t* out_dst[kMaxOutDst];
  int32_t n_heads;              // query heads (units: entry x head x row pair)
  int32_t n_pairs;              // 256-row query blocks per entry (the longest entry's)
  int32_t n_units;              // n_entries * n_heads * n_pairs
  int32_t group;                // num_q_heads / num_kv_heads
  float scale_log2;             // softmax_scale * log2(e)
  int32_t* status;              // device status word
  uint64_t wait_limit_ns;
  int32_t test_stall;           // test hook: the MMA warp first waits on a barrier nothing arrives at
};

template <int D>
struct SmemLayout {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr uint32_t kSub = kBlockM * 128;  // one 64-column (128 B) swizzled sub-tile
  static constexpr uint32_t kQTile = kBlockM * D * 2;
  static constexpr uint32_t kKVTile = kBlockN * D * 2;
  static constexpr uint32_t kPTile = kBlockM * kBlockN * 2;
  static constexpr int kPBufs = D == 128 ? 1 : 2;                    // P buffers (shared by both tiles when 1)
  static constexpr uint32_t kQ = 0;                                  // + tile * kQTile
  static constexpr uint32_t kK = kQ + kTilesPerCta * kQTile;         // + stage * kKVTile
  static constexpr uint32_t kV = kK + kKStages * kKVTile;            // + stage * kKVTile
  static constexpr uint32_t kP = kV + kVStages * kKVTile;            // + buffer * kPTile
  static constexpr uint32_t kBar = kP + kPBufs * kPTile;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bKFull = 1;                      // + stage
  static constexpr int bKEmpty = bKFull + kKStages;     // + stage
  static constexpr int bVFull = bKEmpty + kKStages;     // + stage
  static constexpr int bVEmpty = bVFull + kVStages;     // + stage
  static constexpr int bSFull = bVEmpty + kVStages;     // + tile: S_X(j) is in TMEM
  static constexpr int bSFree = bSFull + kTilesPerCta;  // + tile: softmax X has read S_X(j)
  static constexpr int bPFull = bSFree + kTilesPerCta;  // + tile: P_X(j) is in shared memory
  static constexpr int bPFree = bPFull + kTilesPerCta;  // shared P buffer: the PV MMA reading it finished
  static constexpr int bOReady = bPFree + 1;            // + tile: PV_X(j) finished
  static constexpr int bMmaDone = bOReady + kTilesPerCta;
  static constexpr int kNumBars = bMmaDone + 1;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kEnd = kMisc + 16;
  // +1024 slack to align the dynamic base; at least ~116 KB so one CTA per SM
  // (the CTA allocates all 512 TMEM columns).
  static constexpr uint32_t kAlloc = (kEnd + 1024) > 120 * 1024 ? (kEnd + 1024) : 120 * 1024;
  static_assert(kAlloc <= 232448, "shared memory per CTA");
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

  // Warp-uniform form: every lane waits; true only if all lanes saw the phase.
  __device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity) const {
    return __all_sync(0xffffffffu, wait(bar, parity));
  }

  // Wait for this CTA's own asynchronous work (copies, MMAs) to land before
  // its shared memory or TMEM is released: ignores the abort flag, still
  // bounded by the time limit.
  __device__ __forceinline__ void drain_warp(uint32_t bar, uint32_t parity) const {
    bool done = skptx::mbar_try_wait(bar, parity);
    const uint64_t t0 = skptx::globaltimer_ns();
    while (!done && skptx::globaltimer_ns() - t0 <= limit_ns) done = skptx::mbar_try_wait(bar, parity);
    if (!done) atomicOr(status, kStatusTimeout);
    __syncwarp();
  }
};

// Address of output row `row` of entry `bl`, query head `hq` (kScatter: the
// row's destination buffer, see AttnParams::out_chunk).
template <bool kScatter>
__device__ __forceinline__ uint16_t* out_row_ptr(const AttnParams& p, int bl, int hq, int row) {
  const int64_t head = static_cast<int64_t>(hq) * p.out_sh;
  if constexpr (!kScatter) {
    return p.out + p.out_off[bl] + head + static_cast<int64_t>(row) * p.out_ss;
  } else {
    const int rk = row / p.out_chunk;
    return p.out_dst[rk] + p.out_off[bl] + head + static_cast<int64_t>(row - rk * p.out_chunk) * p.out_ss;
  }
}

template <bool kScatter>
__device__ __forceinline__ void store_zero_rows(const AttnParams& p, int bl, int hq, int r_begin,
                                                int r_end, int D, int tid, int nthreads) {
  const int chunks = D / 8;  // 16-byte chunks per row
  const int total = (r_end - r_begin) * chunks;
  for (int idx = tid; idx < total; idx += nthreads) {
    const int r = r_begin + idx / chunks;
    const int c = idx % chunks;
    *reinterpret_cast<uint4*>(out_row_ptr<kScatter>(p, bl, hq, r) + c * 8) = make_uint4(0, 0, 0, 0);
  }
}

// Valid keys in KV tile j (prefix tiles first, then suffix tiles).
__device__ __forceinline__ int tile_valid(int j, int tP, int nkp, int nks) {
  return (j < tP) ? min(kBlockN, nkp - j * kBlockN) : min(kBlockN, nks - (j - tP) * kBlockN);
}

// Descriptor arithmetic: a shared-memory matrix descriptor holds (address >> 4)
// in its low 14 bits; every operand here lies below 228 KB, so advancing an
// operand by `bytes` is a plain add of bytes >> 4 (no carry leaves the field).
// The issue loops below therefore do one add per MMA on precomputed bases.

// S = Q K^T: 128 x 128 x D, both operands K-major, 128-byte swizzle; the
// K-loop walks 16 columns (32 B) inside a 64-column sub-tile, then the next one.
// Warp-collective (one elected lane issues).
template <int D>
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc) {
  using L = SmemLayout<D>;
  constexpr uint32_t idS = skptx::idesc_bf16_f32(kBlockM, kBlockN, false);
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    const uint64_t off = ((k / 4) * L::kSub + (k % 4) * 32) >> 4;
    skptx::mma_ss_elect(d_tmem, q_desc + off, k_desc + off, idS, k > 0 ? 1u : 0u);
  }
}

// O += P V: P (128 x 128 bf16, K-major, 128-byte swizzle) and V (MN-major,
// head_dim contiguous) from shared memory; each K step covers 16 keys: 32 B of
// a P row and 2048 B of V rows.  Warp-collective.
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint64_t p_desc, uint64_t v_desc, bool accumulate) {
  using L = SmemLayout<D>;
  constexpr uint32_t idO = skptx::idesc_bf16_f32(kBlockM, D, true);
#pragma unroll
  for (int k = 0; k < kBlockN / 16; ++k) {
    const uint64_t poff = ((k / 4) * L::kSub + (k % 4) * 32) >> 4;
    skptx::mma_ss_elect(o_tmem, p_desc + poff, v_desc + ((k * 2048) >> 4), idO,
                        (accumulate || k > 0) ? 1u : 0u);
  }
}

// Exponentiate one tile row, sum it, and pack P as bf16 pairs.  PARTIAL:
// columns >= nvalid are exact zeros (only the last tile of each source can be
// partial; full tiles take the select-free path).
template <bool PARTIAL>
__device__ __forceinline__ float exp_row_pack(const float (&s)[kBlockN], float sl2, float neg_m, int nvalid,
                                              uint32_t (&pk)[kBlockN / 2]) {
  float sum8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) sum8[i] = 0.f;
#pragma unroll
  for (int c = 0; c < kBlockN; c += 2) {
    float e0 = skptx::ex2_approx(fmaf(s[c], sl2, neg_m));
    float e1 = skptx::ex2_approx(fmaf(s[c + 1], sl2, neg_m));
    // exact zeros for masked columns (also when scale == 0, where -inf * 0 is NaN)
    if (PARTIAL && c >= nvalid) e0 = 0.f;
    if (PARTIAL && c + 1 >= nvalid) e1 = 0.f;
    sum8[c % 8] += e0;
    sum8[(c + 1) % 8] += e1;
    pk[c / 2] = skptx::pack_bf16x2(e0, e1);
  }
  return ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
}

// Store one P row (128 bf16 = 16 chunks of 16 B) of a K-major 128-byte-swizzled
// tile: chunk q of row r goes to sub-tile q / 8, position (q % 8) ^ (r % 8).
__device__ __forceinline__ void store_p_row(uint32_t p_base, int r, const uint32_t (&pk)[kBlockN / 2]) {
  const uint32_t row = p_base + static_cast<uint32_t>(r) * 128u;
  const uint32_t sw = static_cast<uint32_t>(r & 7);
#pragma unroll
  for (int q = 0; q < kBlockN / 8; ++q) {
    const uint32_t addr = row + (q / 8) * (kBlockM * 128u) + ((static_cast<uint32_t>(q % 8) ^ sw) << 4);
    skptx::st_shared_v4(addr, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  }
}

template <int D, bool kScatter = false>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using L = SmemLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = skptx::smem_addr(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  const int hq = blockIdx.y;
  const int bl = blockIdx.z;
  const int row0 = blockIdx.x * kRowsPerCta;
  const int qv = p.q_valid[bl];
  const int nkp = p.n_prefix[bl];
  const int nks = p.n_suffix[bl];
  const int tP = (nkp + kBlockN - 1) / kBlockN;
  const int tS = (nks + kBlockN - 1) / kBlockN;
  const int n_tiles = tP + tS;
  const int sq = p.sq[bl];
  uint16_t* out_bh = p.out + p.out_off[bl] + static_cast<int64_t>(hq) * p.out_sh;  // plain output only

  if (row0 >= qv || n_tiles == 0) {
    // Every row of this CTA is pad, or this batch row has no valid key: exact zeros.
    const int r_end = min(row0 + kRowsPerCta, sq);
    store_zero_rows<kScatter>(p, bl, hq, row0, r_end, D, threadIdx.x, kThreads);
    return;
  }

  auto bar = [&](int i) -> uint32_t { return sbase + L::kBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  if (threadIdx.x == 0) {
    skptx::mbar_init(bar(L::bQFull), 1);
    for (int s = 0; s < kKStages; ++s) {
      skptx::mbar_init(bar(L::bKFull + s), 1);
      skptx::mbar_init(bar(L::bKEmpty + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      skptx::mbar_init(bar(L::bVFull + s), 1);
      skptx::mbar_init(bar(L::bVEmpty + s), 1);
    }
    for (int x = 0; x < kTilesPerCta; ++x) {
      skptx::mbar_init(bar(L::bSFull + x), 1);
      skptx::mbar_init(bar(L::bSFree + x), kBlockM);
      skptx::mbar_init(bar(L::bPFull + x), kBlockM);
      skptx::mbar_init(bar(L::bOReady + x), 1);
    }
    skptx::mbar_init(bar(L::bPFree), 1);
    skptx::mbar_init(bar(L::bMmaDone), 1);
    *abort_flag = 0;
    skptx::fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    skptx::tmem_alloc(skptx::smem_addr(tmem_slot), kTmemCols);
    skptx::tmem_relinquish();
  }
  skptx::tc_fence_before();
  __syncthreads();
  skptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, p.status, p.wait_limit_ns};

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    const int hkv = hq / p.group;
    if (lane == 0) {
      skptx::prefetch_tmap(&p.tm_q[bl]);
      if (tP > 0) { skptx::prefetch_tmap(&p.tm_kp[bl]); skptx::prefetch_tmap(&p.tm_vp[bl]); }
      if (tS > 0) { skptx::prefetch_tmap(&p.tm_ks[bl]); skptx::prefetch_tmap(&p.tm_vs[bl]); }
    }
    __syncwarp();
    skptx::mbar_arrive_expect_tx_elect(bar(L::bQFull), kTilesPerCta * L::kQTile);
#pragma unroll
    for (int x = 0; x < kTilesPerCta; ++x)
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        skptx::tma_load_3d_elect(sbase + L::kQ + x * L::kQTile + c * L::kSub, &p.tm_q[bl], bar(L::bQFull),
                                 c * 64, hq, row0 + x * kBlockM);
    // Load order K0, K1, V0, K2, V1, ...: K(j+1) is needed (by S(j+1)) before V(j).
    int jk = 0, jv = 0;
    bool ok = true;
    while (ok && (jk < n_tiles || jv < n_tiles)) {
      const bool do_k = jk < n_tiles && jk <= jv + 1;
      const int j = do_k ? jk : jv;
      const bool pre = j < tP;
      const int key0 = (pre ? j : j - tP) * kBlockN;
      if (do_k) {
        const int s = j % kKStages;
        if (j >= kKStages && !W.wait_warp(bar(L::bKEmpty + s), ((j / kKStages) - 1) & 1)) { ok = false; break; }
        const CUtensorMap* mk = pre ? &p.tm_kp[bl] : &p.tm_ks[bl];
        skptx::mbar_arrive_expect_tx_elect(bar(L::bKFull + s), L::kKVTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          skptx::tma_load_3d_elect(sbase + L::kK + s * L::kKVTile + c * L::kSub, mk, bar(L::bKFull + s),
                                   c * 64, hkv, key0);
        ++jk;
      } else {
        const int s = j % kVStages;
        if (j >= kVStages && !W.wait_warp(bar(L::bVEmpty + s), ((j / kVStages) - 1) & 1)) { ok = false; break; }
        const CUtensorMap* mv = pre ? &p.tm_vp[bl] : &p.tm_vs[bl];
        skptx::mbar_arrive_expect_tx_elect(bar(L::bVFull + s), L::kKVTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          skptx::tma_load_3d_elect(sbase + L::kV + s * L::kKVTile + c * L::kSub, mv, bar(L::bVFull + s),
                                   c * 64, hkv, key0);
        ++jv;
      }
    }
    // Drain: no copy issued by this CTA may still be landing when it exits.
    // On the normal path every wait below has already completed.
    W.drain_warp(bar(L::bQFull), 0);
    for (int j = (jk > kKStages ? jk - kKStages : 0); j < jk; ++j)
      W.drain_warp(bar(L::bKFull + j % kKStages), (j / kKStages) & 1);
    for (int j = (jv > kVStages ? jv - kVStages : 0); j < jv; ++j)
      W.drain_warp(bar(L::bVFull + j % kVStages), (j / kVStages) & 1);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t dQ = skptx::sdesc_sw128(sbase + L::kQ, 16, 1024);
    const uint64_t dK = skptx::sdesc_sw128(sbase + L::kK, 16, 1024);
    const uint64_t dV = skptx::sdesc_sw128(sbase + L::kV, L::kSub, 1024);
    const uint64_t dP = skptx::sdesc_sw128(sbase + L::kP, 16, 1024);
    bool ok = W.wait_warp(bar(L::bQFull), 0) && W.wait_warp(bar(L::bKFull), 0);
    // Test hook for the bounded-wait path: MmaDone is only committed by this
    // warp after its loop, so this wait runs out (every role then aborts,
    // drains and exits with SK_ERR_DEVICE_TIMEOUT in the status word).
    if (p.test_stall) ok = ok && W.wait_warp(bar(L::bMmaDone), 0);
    if (ok) {
      skptx::tc_fence_after();
#pragma unroll
      for (int x = 0; x < kTilesPerCta; ++x) {
        issue_s<D>(tmem + x * 128, dQ + ((x * L::kQTile) >> 4), dK);
        skptx::mma_commit_elect(bar(L::bSFull + x));
      }
      skptx::mma_commit_elect(bar(L::bKEmpty));
    }
    // Each tile has two in-order streams, S_X(1..n-1) and PV_X(0..n-1); any op
    // whose inputs are ready is issued, so neither tile's progress waits for
    // the other's.  A K (V) stage is released once both tiles' S (PV) MMAs
    // reading it are issued (the commit fires when they complete).
    // Warp-uniform readiness: every lane probes, all must agree (else retry).
    auto ready = [](uint32_t b, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, skptx::mbar_test_wait(b, parity));
    };
    int sN[kTilesPerCta], pN[kTilesPerCta];
#pragma unroll
    for (int x = 0; x < kTilesPerCta; ++x) { sN[x] = 1; pN[x] = 0; }
    uint64_t stall_t0 = 0;
    uint32_t spins = 0;
    while (ok && (pN[0] < n_tiles || pN[1] < n_tiles)) {
      bool progressed = false;
#pragma unroll
      for (int x = 0; x < kTilesPerCta; ++x) {
        const int o = 1 - x;
        const int j = pN[x];
        if (j < n_tiles && ready(bar(L::bPFull + x), j & 1) &&
            ready(bar(L::bVFull + j % kVStages), (j / kVStages) & 1)) {
          skptx::tc_fence_after();
          const int b = x % L::kPBufs;
          issue_pv<D>(tmem + 256 + x * 128, dP + ((b * L::kPTile) >> 4),
                      dV + (((j % kVStages) * L::kKVTile) >> 4), j > 0);
          skptx::mma_commit_elect(bar(L::bOReady + x));
          if (L::kPBufs == 1) skptx::mma_commit_elect(bar(L::bPFree));
          if (pN[o] > j) skptx::mma_commit_elect(bar(L::bVEmpty + j % kVStages));
          pN[x] = j + 1;
          progressed = true;
        }
        const int k = sN[x];
        if (k < n_tiles && ready(bar(L::bSFree + x), (k - 1) & 1) &&
            ready(bar(L::bKFull + k % kKStages), (k / kKStages) & 1)) {
          skptx::tc_fence_after();
          issue_s<D>(tmem + x * 128, dQ + ((x * L::kQTile) >> 4), dK + (((k % kKStages) * L::kKVTile) >> 4));
          skptx::mma_commit_elect(bar(L::bSFull + x));
          if (sN[o] > k) skptx::mma_commit_elect(bar(L::bKEmpty + k % kKStages));
          sN[x] = k + 1;
          progressed = true;
        }
      }
      // Bounded: give up once nothing has become ready for the wait limit.
      if (progressed) {
        spins = 0;
      } else if (spins++ == 0) {
        stall_t0 = skptx::globaltimer_ns();
      } else if ((spins & 31u) == 0) {
        if (*abort_flag) ok = false;
        else if (skptx::globaltimer_ns() - stall_t0 > p.wait_limit_ns) {
          *abort_flag = 1;
          atomicOr(p.status, kStatusTimeout);
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok);
      }
    }
    // Every MMA this warp issued has finished before TMEM is released.
    skptx::mma_commit_elect(bar(L::bMmaDone));
    W.drain_warp(bar(L::bMmaDone), 0);
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int x = warp / 4;            // query tile of this warpgroup
    const int r = threadIdx.x % 128;   // row in tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS_ = tmem + lane_base + static_cast<uint32_t>(x) * 128;
    const uint32_t tO = tmem + lane_base + 256 + static_cast<uint32_t>(x) * 128;
    const int pb = x % L::kPBufs;
    const uint32_t p_base = sbase + L::kP + pb * L::kPTile;
    const float sl2 = p.scale_log2;
    float m_run = 0.f;  // running (possibly stale) max of scale*log2(e)*s
    float l_run = 0.f;  // running sum of exponentials
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = W.wait_warp(bar(L::bSFull + x), j & 1);
      if (!ok) break;
      skptx::tc_fence_after();
      float s[kBlockN];
      {
        uint32_t u[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) skptx::tmem_ld32(tS_ + c * 32, u[c]);
        skptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) skptx::reg_fence(u[c]);
#pragma unroll
        for (int c = 0; c < kBlockN; ++c) s[c] = __uint_as_float(u[c / 32][c % 32]);
      }
      // S_X(j) is in registers: the issuer may overwrite it with S_X(j+1).
      skptx::tc_fence_before();
      skptx::mbar_arrive(bar(L::bSFree + x));
      const int nvalid = tile_valid(j, tP, nkp, nks);
      const bool partial = nvalid < kBlockN;
      if (partial) {
#pragma unroll
        for (int c = 0; c < kBlockN; ++c)
          if (c >= nvalid) s[c] = -INFINITY;
      }
      // row max with 8 independent chains
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
      for (int c = 8; c < kBlockN; ++c) mx8[c % 8] = fmaxf(mx8[c % 8], s[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_tile = mx * sl2;
      float alpha = 1.f;
      bool raise = false;
      if (j == 0) {
        m_run = m_tile;
      } else if (m_tile > m_run + kRescaleLog2) {
        alpha = skptx::ex2_approx(m_run - m_tile);
        m_run = m_tile;
        raise = true;
      }
      uint32_t pk[kBlockN / 2];
      const float sum = partial ? exp_row_pack<true>(s, sl2, -m_run, nvalid, pk)
                                : exp_row_pack<false>(s, sl2, -m_run, nvalid, pk);
      l_run = l_run * alpha + sum;
      // Before P_X(j) is stored and before O_X is touched, PV_X(j-1) must have
      // finished.  This also keeps every barrier below within one phase of
      // its waiter (a parity wait cannot tell phase k from k+2).
      if (j > 0) {
        ok = W.wait_warp(bar(L::bOReady + x), (j - 1) & 1);
        if (!ok) break;
      }
      if (L::kPBufs == 1) {
        // One P buffer for both tiles, used in the order A(0), B(0), A(1), ...:
        // use u may start once the PV MMA of use u-1 has finished.
        const int use = 2 * j + x;
        if (use > 0) {
          ok = W.wait_warp(bar(L::bPFree), (use - 1) & 1);
          if (!ok) break;
        }
      }
      store_p_row(p_base, r, pk);
      if (__any_sync(0xffffffffu, raise)) {
        // O holds the sum over tiles < j with the old max (PV_X(j) waits for
        // this thread's arrive below).
        skptx::tc_fence_after();
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
        skptx::tmem_wait_st();
      }
      skptx::fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
      skptx::tc_fence_before();
      skptx::mbar_arrive(bar(L::bPFull + x));
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = W.wait_warp(bar(L::bOReady + x), (n_tiles - 1) & 1);
    if (ok) {
      skptx::tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      const int row = row0 + x * kBlockM + r;
      uint16_t* orow = kScatter ? out_row_ptr<true>(p, bl, hq, row < sq ? row : 0)
                                : out_bh + static_cast<int64_t>(row) * p.out_ss;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        skptx::tmem_ld32(tO + c * 32, o);
        skptx::tmem_wait_ld();
        skptx::reg_fence(o);
        if (row < sq) {
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
  if (warp == kMmaWarp) {
    skptx::tc_fence_after();
    skptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace skattn
