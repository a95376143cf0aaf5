// Fused Q/K RMSNorm + RoPE prologue, in place ("vLLM-Omni performance
// patterns", Q/K RMSNorm + RoPE section; "sglang PR 26973", cosmos3video.py).
//
// Memory-bound: one pass reads and writes every q/k element once.  A row is
// one (token, head) vector of D bf16 values handled by D/8 threads, each with
// one 16-byte load and one 16-byte store.  The sum of squares is reduced with
// xor-shuffles inside the row's lane group; in half-split (NeoX) mode the
// rotation partner (d + rot_dim/2) lives rot_dim/16 lanes away and is fetched
// with one shuffle of the already bf16-rounded normalised values.
// Rounding follows the unfused path: RMSNorm output rounded to bf16, rotation
// in fp32, result rounded to bf16 (nearest even).
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

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float round_bf16(float x) {
  uint32_t r = pack2(x, 0.f);
  return bf16lo(r);
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
  float x[8], wf[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = bf16lo(xw[i]);
    x[2 * i + 1] = bf16hi(xw[i]);
    wf[2 * i] = bf16lo(ww[i]);
    wf[2 * i + 1] = bf16hi(ww[i]);
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
#pragma unroll
  for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss * (1.0f / D) + p.eps);
  float y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = round_bf16(x[i] * r * wf[i]);

  const int d0 = sub * 8;
  const int rot = p.rot_dim;
  float z[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) z[i] = y[i];

  if (p.interleaved) {
    if (valid && d0 < rot) {
      const float* crow = p.table + static_cast<int64_t>(s) * rot;
      const float4 c4 = *reinterpret_cast<const float4*>(crow + d0 / 2);
      const float4 s4 = *reinterpret_cast<const float4*>(crow + rot / 2 + d0 / 2);
      const float cs[4] = {c4.x, c4.y, c4.z, c4.w};
      const float sn[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = y[2 * e], c = y[2 * e + 1];
        z[2 * e] = fmaf(a, cs[e], -(c * sn[e]));
        z[2 * e + 1] = fmaf(c, cs[e], a * sn[e]);
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
    for (int i = 0; i < 4; ++i) yp[i] = __shfl_sync(0xffffffffu, pack2(y[2 * i], y[2 * i + 1]), src);
    if (valid && (first || second)) {
      float ypart[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ypart[2 * i] = bf16lo(yp[i]);
        ypart[2 * i + 1] = bf16hi(yp[i]);
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
        for (int e = 0; e < 8; ++e) z[e] = fmaf(y[e], cs[e], -(ypart[e] * sn[e]));
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) z[e] = fmaf(y[e], cs[e], ypart[e] * sn[e]);
      }
    }
  }
  if (valid) {
    uint4 o;
    o.x = pack2(z[0], z[1]);
    o.y = pack2(z[2], z[3]);
    o.z = pack2(z[4], z[5]);
    o.w = pack2(z[6], z[7]);
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
