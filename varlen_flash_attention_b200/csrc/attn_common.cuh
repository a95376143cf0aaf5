// Definitions shared by the attention kernels: tile sizes, the launch
// parameters of the split-KV form, the bounded barrier wait, output row
// addressing.
//
// The operation ("sglang PR 26973", forward_with_replicated_kv_prefix;
// "sglang PR 30107", tail_attn_meta / tail-pad layout invariant):
//   O = softmax(scale * Q K*^T) V*,  K*/V* = cat(prefix, suffix)[0:real_len]
// for each batch row and query head, query head h reading KV head
// h / (num_q_heads / num_kv_heads); query rows past q_valid and all rows of a
// row block with no valid key are written as zeros.
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

// Valid keys in KV tile j (prefix tiles first, then suffix tiles).
__device__ __forceinline__ int tile_valid(int j, int tP, int nkp, int nks) {
  return (j < tP) ? min(kBlockN, nkp - j * kBlockN) : min(kBlockN, nks - (j - tP) * kBlockN);
}

}  // namespace skattn
