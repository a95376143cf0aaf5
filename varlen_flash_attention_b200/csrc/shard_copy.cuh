// Tail-padded shard copy ("sglang PR 30107", shard_like: pad the stream's tail
// with num_pad rows, zeros or repeats of the last row, then take one rank's
// local_len rows), fused into one pass that reads only this rank's real rows.
// Only the last rank of a tail-padded shard needs a copy at all (every other
// rank's chunk is a view of the input); the pages' cat+pad kernel for the
// same kind of step copies 16-byte chunks ("sglang PR 29281"), as this does.
//
// HBM-bound: every destination byte is written once, every real source row
// of the chunk read once.  One thread per 16-byte chunk, grid-stride.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace skshard {

struct PadCopyParams {
  const uint8_t* src;
  uint8_t* dst;
  int64_t src_sb, src_ss;  // bytes
  int64_t dst_sb, dst_ss;  // bytes
  int32_t src_rows;        // rows of the (unpadded) source stream
  int32_t dst_rows;        // rows of the destination chunk (local_len)
  int32_t first_row;       // source row of destination row 0 (rank * local_len)
  int32_t row_chunks;      // 16-byte chunks per row
  int32_t batch;
  int32_t repeat_last;     // pad rows repeat the last source row instead of zeros
};

__global__ void __launch_bounds__(256) pad_copy_kernel(const PadCopyParams p) {
  const int64_t per_b = static_cast<int64_t>(p.dst_rows) * p.row_chunks;
  const int64_t total = per_b * p.batch;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / per_b;
    const int64_t rem = i - b * per_b;
    const int r = static_cast<int>(rem / p.row_chunks);
    const int c = static_cast<int>(rem - static_cast<int64_t>(r) * p.row_chunks);
    int s = p.first_row + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (s >= p.src_rows && p.repeat_last) s = p.src_rows - 1;
    if (s < p.src_rows)
      v = *reinterpret_cast<const uint4*>(p.src + b * p.src_sb + static_cast<int64_t>(s) * p.src_ss + c * 16);
    *reinterpret_cast<uint4*>(p.dst + b * p.dst_sb + static_cast<int64_t>(r) * p.dst_ss + c * 16) = v;
  }
}

}  // namespace skshard
