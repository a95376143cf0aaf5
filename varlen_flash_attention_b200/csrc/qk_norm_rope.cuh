// Fused Q/K RMSNorm + RoPE prologue, in place ("vLLM-Omni performance
// patterns", Q/K RMSNorm + RoPE section; "sglang PR 26973", cosmos3video.py).
//
// Memory-bound: one pass reads and writes every q/k element once.  A row is
// one (token, head) vector of D bf16 values handled by D/8 threads, each with
// one 16-byte load and one 16-byte store.  The sum of squares is reduced with
// xor-shuffles inside the row's lane group; in half-split (NeoX) mode the
// rotation partner (d + rot_dim/2) lives rot_dim/16 lanes away and is fetched
// with one shuffle of the already bf16-rounded normalised values.
// Rounding follows the unfused path: RMSNorm output rounded to bf16, rotation,
// result rounded to bf16 (nearest even).  The arithmetic is fp64: the kernel is
// bound by HBM, and in fp64 every product of a bf16 value with an fp32 table
// entry is exact, so the one rounding before each bf16 store is the only one
// that matters (fp32 is not enough when the rotation cancels).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace skqkn {

struct NormRopeParams {
  uint16_t* q;
  uint16_t* k;
  int64_t q_sb, q_ss, q_sh;
  int64_t k_sb, k_ss, k_sh;
  const uint16_t* w_q;
  const uint16_t* w_k;
  const float* table;  // [rows, rot_dim] = [cos | sin]
  int rot_dim;
  bool interleaved;
  float eps;
  int S, Hq, Hkv, B;
};

// Nearest-even bf16 of a double, rounded once: through fp32 (nearest), then to
// bf16, correcting the one case where the fp32 step lands exactly on a bf16
// midpoint that the double was not on.
__device__ __forceinline__ uint32_t bf16_bits_rn(double x) {
  const float f = __double2float_rn(x);
  const uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u) return (u & 0x7FFFFFFFu) > 0x7F800000u ? 0x7FC0u : (u >> 16);
  uint32_t up = u >> 16;
  const uint32_t low = u & 0xFFFFu;
  if (low > 0x8000u) {
    up += 1;
  } else if (low == 0x8000u) {
    const double fd = static_cast<double>(f);
    if (fd == x) up += (up & 1u);
    else if (fabs(x) > fabs(fd)) up += 1;
  }
  return up;
}

__device__ __forceinline__ double bf16_to_f64(uint32_t bits16) {
  return static_cast<double>(__uint_as_float(bits16 << 16));
}

template <int D>
__global__ void __launch_bounds__(256) qk_norm_rope_kernel(const NormRopeParams p) {
  constexpr int TPR = D / 8;      // threads per row
  constexpr int RPB = 256 / TPR;  // rows per block
  const int H = p.Hq + p.Hkv;
  const int64_t total = static_cast<int64_t>(p.B) * p.S * H;
  const int sub = threadIdx.x % TPR;
  const int lane = threadIdx.x % 32;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * RPB + threadIdx.x / TPR;
  const bool valid = row < total;

  int head = 0, s = 0, b = 0;
  if (valid) {
    head = static_cast<int>(row % H);
    const int64_t tok = row / H;
    s = static_cast<int>(tok % p.S);
    b = static_cast<int>(tok / p.S);
  }
  const bool is_q = head < p.Hq;
  uint16_t* ptr = is_q ? p.q + b * p.q_sb + s * p.q_ss + static_cast<int64_t>(head) * p.q_sh
                       : p.k + b * p.k_sb + s * p.k_ss + static_cast<int64_t>(head - p.Hq) * p.k_sh;
  ptr += sub * 8;
  const uint16_t* w = (is_q ? p.w_q : p.w_k) + sub * 8;

  uint4 xv = make_uint4(0, 0, 0, 0);
  uint4 wv = make_uint4(0, 0, 0, 0);
  if (valid) {
    xv = *reinterpret_cast<const uint4*>(ptr);
    wv = *reinterpret_cast<const uint4*>(w);
  }
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
  const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
  double x[8], wf[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = bf16_to_f64(xw[i] & 0xFFFFu);
    x[2 * i + 1] = bf16_to_f64(xw[i] >> 16);
    wf[2 * i] = bf16_to_f64(ww[i] & 0xFFFFu);
    wf[2 * i + 1] = bf16_to_f64(ww[i] >> 16);
  }
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss += x[i] * x[i];
#pragma unroll
  for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const double r = 1.0 / sqrt(ss / static_cast<double>(D) + static_cast<double>(p.eps));
  uint32_t yb[8];
  double y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    yb[i] = bf16_bits_rn(x[i] * r * wf[i]);
    y[i] = bf16_to_f64(yb[i]);
  }

  const int d0 = sub * 8;
  const int rot = p.rot_dim;
  uint32_t zb[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) zb[i] = yb[i];

  if (p.interleaved) {
    if (valid && d0 < rot) {
      const float* crow = p.table + static_cast<int64_t>(s) * rot;
      const float4 c4 = *reinterpret_cast<const float4*>(crow + d0 / 2);
      const float4 s4 = *reinterpret_cast<const float4*>(crow + rot / 2 + d0 / 2);
      const float cs[4] = {c4.x, c4.y, c4.z, c4.w};
      const float sn[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double a = y[2 * e], c = y[2 * e + 1];
        zb[2 * e] = bf16_bits_rn(a * static_cast<double>(cs[e]) - c * static_cast<double>(sn[e]));
        zb[2 * e + 1] = bf16_bits_rn(c * static_cast<double>(cs[e]) + a * static_cast<double>(sn[e]));
      }
    }
  } else {
    const int half = rot / 2;
    const int hs = half / 8;  // partner lane distance
    const bool first = d0 < half;
    const bool second = !first && d0 < rot;
    const int psub = first ? sub + hs : (second ? sub - hs : sub);
    const int src = (lane & ~(TPR - 1)) + psub;
    uint32_t yp[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) yp[i] = __shfl_sync(0xffffffffu, yb[2 * i] | (yb[2 * i + 1] << 16), src);
    if (valid && (first || second)) {
      double ypart[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ypart[2 * i] = bf16_to_f64(yp[i] & 0xFFFFu);
        ypart[2 * i + 1] = bf16_to_f64(yp[i] >> 16);
      }
      const int i0 = first ? d0 : d0 - half;
      const float* crow = p.table + static_cast<int64_t>(s) * rot;
      const float4 c0 = *reinterpret_cast<const float4*>(crow + i0);
      const float4 c1 = *reinterpret_cast<const float4*>(crow + i0 + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(crow + half + i0);
      const float4 s1 = *reinterpret_cast<const float4*>(crow + half + i0 + 4);
      const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      if (first) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          zb[e] = bf16_bits_rn(y[e] * static_cast<double>(cs[e]) - ypart[e] * static_cast<double>(sn[e]));
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          zb[e] = bf16_bits_rn(y[e] * static_cast<double>(cs[e]) + ypart[e] * static_cast<double>(sn[e]));
      }
    }
  }
  if (valid) {
    uint4 o;
    o.x = zb[0] | (zb[1] << 16);
    o.y = zb[2] | (zb[3] << 16);
    o.z = zb[4] | (zb[5] << 16);
    o.w = zb[6] | (zb[7] << 16);
    *reinterpret_cast<uint4*>(ptr) = o;
  }
}

inline cudaError_t launch(const NormRopeParams& p, int D, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(p.B) * p.S * (p.Hq + p.Hkv);
  const int tpr = D / 8;
  const int rpb = 256 / tpr;
  const int64_t blocks = (total + rpb - 1) / rpb;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  if (blocks == 0) return cudaSuccess;
  switch (D) {
    case 64: qk_norm_rope_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p); break;
    case 128: qk_norm_rope_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p); break;
    case 256: qk_norm_rope_kernel<256><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace skqkn
