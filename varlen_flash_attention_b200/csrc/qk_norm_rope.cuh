// Fused Q/K RMSNorm + RoPE prologue, in place ("vLLM-Omni performance
// patterns", Q/K RMSNorm + RoPE section; "sglang PR 26973", cosmos3video.py).
//
// One pass reads and writes every q/k element once.  A row is one (token,
// head) vector of D bf16 values handled by D/8 lanes, 8 dims each, with one
// 16-byte load and one 16-byte store.  The sum of squares is reduced with
// xor-shuffles inside the row's lane group; in half-split (NeoX) mode the
// rotation partner (d + rot_dim/2) lives rot_dim/16 lanes away and is fetched
// with one shuffle of the already bf16-rounded normalised values.
//
// Two instances.  The default (qk_norm_rope_warp_kernel) evaluates the
// unfused path in fp32 with its two bf16 rounding points: the sum of squares
// and r = rsqrt(mean + eps) in fp32, y = bf16(x * r * w), then the rotation
// z = bf16(y * cos -/+ y_partner * sin) with one fused multiply-add; about ten
// instructions per element, so the kernel is bound by HBM.  Each result is
// within three bf16 ulps, at the magnitude of its own two rotation terms, of
// the formula evaluated exactly (the bound is derived in the tests).
//
// The exact instance (qk_norm_rope_kernel) returns the bits of the unfused
// path computed in fp64: r = 1/sqrt(mean
// x^2 + eps) in fp64, y = bf16(x * r * w) with both products rounded in fp64,
// z = bf16 of the rotation evaluated in fp64 (products of a bf16 value and an
// fp32 table entry are exact there).  The kernel reaches the same bits with
// fp32 arithmetic for y and z: each fp32 result carries a proven error bound
// of a few fp32 ulps, so its bf16 rounding is the fp64 one unless it lies
// within that bound of a bf16 midpoint; those elements (about 3 in 10^4), and
// rows outside the ranges the bounds assume, are recomputed in fp64.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
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

// fp32 bits -> bf16 pair, nearest even (low half from lo, high half from hi).
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// True when the bf16 rounding of an fp32 value known only to within 4 fp32
// ulps is undecided: its low 16 bits are within 4 of the midpoint 0x8000.
__device__ __forceinline__ bool near_bf16_midpoint(float v) {
  return ((__float_as_uint(v) & 0xFFFFu) - 0x7FFCu) <= 8u;
}

// y = x * r * w in fp32 with r_f the fp32 rounding of the fp64 r: three fp32
// roundings, so |y32 - y64| <= 3.0001 * 2^-24 |y| <= 3.0001 fp32 ulps of y32.
// Flags a midpoint case, and 0 < |y| < 2^-60 (below that the partner products
// of the rotation could leave fp32's normal range).
__device__ __forceinline__ float norm_fp32(float x, float r_f, float w, bool& flag) {
  const float y = __fmul_rn(__fmul_rn(x, r_f), w);
  const uint32_t mag = __float_as_uint(y) & 0x7FFFFFFFu;
  flag = flag || near_bf16_midpoint(y) || (mag - 1u) < 0x217FFFFFu;
  return y;
}

// z = y * c + yp * sg in fp32: yp * sg split exactly into q + qe (fma), the
// rest with two roundings; |z32 - z| <= 2.01 * 2^-24 |z| (<= 2.01 ulps) as long
// as |z32| >= 2^-16 |q| (cancellation beyond that is flagged).  y, yp are bf16
// values, c and sg fp32 values.  A zero result carries the sign the fp64
// evaluation gives it: qe is -0 whenever yp * sg is a zero, so z = t exactly.
__device__ __forceinline__ float rot_fp32(float y, float yp, float c, float sg, bool& flag) {
  const float q = __fmul_rn(yp, sg);
  const float qe = -__fmaf_rn(-yp, sg, q);  // yp * sg - q, and -0 when yp * sg is a zero
  const float t = __fmaf_rn(y, c, q);
  const float z = __fadd_rn(t, qe);
  flag = flag || near_bf16_midpoint(z) || fabsf(z) * 65536.0f < fabsf(q);
  return z;
}

// One lane's 8 dims of one row, the oracle's operations one by one in fp64
// (the general path: subnormal, overflowing and non-finite values, and rows
// whose ranges the fp32 bounds do not cover).  z_i = y_i * c_i + y_partner *
// sg_i, sg carrying the rotation's sign; lanes past rot_dim pass y through.
__device__ __forceinline__ uint4 row_general(uint4 xv, const float* w, double r, const float* c, const float* sg,
                                             bool interleaved, int src, bool rotates) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
  uint32_t yb[8];
  double y[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    yb[2 * i] = bf16_bits_rn(bf16_to_f64(xw[i] & 0xFFFFu) * r * static_cast<double>(w[2 * i]));
    yb[2 * i + 1] = bf16_bits_rn(bf16_to_f64(xw[i] >> 16) * r * static_cast<double>(w[2 * i + 1]));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = bf16_to_f64(yb[i]);
  double yp[8];
  if (interleaved) {
#pragma unroll
    for (int i = 0; i < 8; ++i) yp[i] = y[i ^ 1];
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t pk = __shfl_sync(0xffffffffu, yb[2 * i] | (yb[2 * i + 1] << 16), src);
      yp[2 * i] = bf16_to_f64(pk & 0xFFFFu);
      yp[2 * i + 1] = bf16_to_f64(pk >> 16);
    }
  }
  uint32_t zb[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    zb[i] = rotates ? bf16_bits_rn(fma(yp[i], static_cast<double>(sg[i]), y[i] * static_cast<double>(c[i])))
                    : yb[i];
  return make_uint4(zb[0] | (zb[1] << 16), zb[2] | (zb[3] << 16), zb[4] | (zb[5] << 16), zb[6] | (zb[7] << 16));
}

// One block = kNormRopeThreads / (D/8) tokens; D/8 lanes own one token and walk all its
// Hq + Hkv rows, 8 dims per lane, so the lane's cos/sin entries are loaded
// once per token and the weights once per block (shared memory).  Rows are
// loaded 2 at a time, one batch ahead.  Per batch: the rows' sums of squares
// in fp64 (exact conversions), one fp64 square root and division per lane
// (lane j of the group takes row j), then per row the fp32 y and rotation
// with exact fp64 fix-ups for flagged lanes.  A row takes the general path
// (warp-wide vote) when r is outside [2^-100, 2^100] (this includes every
// non-finite input and eps = 0 on a zero row) or the lane's weights or table
// entries are outside the ranges the fp32 bounds assume.
constexpr int kNormRopeThreads = 256;
constexpr int kNormRopeMinBlocks = 3;

template <int D>
__global__ void __launch_bounds__(kNormRopeThreads, kNormRopeMinBlocks) qk_norm_rope_kernel(const NormRopeParams p) {
  constexpr int TPR = D / 8;                      // lanes per row
  constexpr int GROUPS = kNormRopeThreads / TPR;  // tokens per block
  constexpr int BATCH = 2;                        // rows per batch
  __shared__ __align__(16) float w_s[2][D];
  for (int i = threadIdx.x; i < 2 * D; i += blockDim.x)
    w_s[i / D][i % D] = __uint_as_float(static_cast<uint32_t>((i < D ? p.w_q : p.w_k)[i % D]) << 16);
  __syncthreads();

  const int sub = threadIdx.x % TPR;
  const int lane = threadIdx.x % 32;
  const int d0 = sub * 8;
  const int64_t tok = static_cast<int64_t>(blockIdx.x) * GROUPS + threadIdx.x / TPR;
  const bool valid = tok < static_cast<int64_t>(p.B) * p.S;
  const int s = valid ? static_cast<int>(tok % p.S) : 0;
  const int b = valid ? static_cast<int>(tok / p.S) : 0;

  // |w| <= 2^30 bounds |y| <= 16 |w| <= 2^34 (|x r| <= sqrt(D) <= 16)
  bool wq_ok = true, wk_ok = true;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    wq_ok = wq_ok && fabsf(w_s[0][d0 + i]) <= 0x1p30f;
    wk_ok = wk_ok && fabsf(w_s[1][d0 + i]) <= 0x1p30f;
  }

  const int rot = p.rot_dim;
  const bool rotates = d0 < rot;
  float c[8], sg[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) { c[i] = 1.0f; sg[i] = 0.0f; }
  int src = lane;
  bool cs_ok = true;
  if (rotates) {
    const float* crow = p.table + static_cast<int64_t>(s) * rot;
    if (p.interleaved) {
      const float4 c4 = *reinterpret_cast<const float4*>(crow + d0 / 2);
      const float4 s4 = *reinterpret_cast<const float4*>(crow + rot / 2 + d0 / 2);
      const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
      const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        c[2 * e] = c[2 * e + 1] = cv[e];
        sg[2 * e] = -sv[e];
        sg[2 * e + 1] = sv[e];
      }
    } else {
      const int half = rot / 2;
      const bool first = d0 < half;
      const int i0 = first ? d0 : d0 - half;
      const float4 c0 = *reinterpret_cast<const float4*>(crow + i0);
      const float4 c1 = *reinterpret_cast<const float4*>(crow + i0 + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(crow + half + i0);
      const float4 s1 = *reinterpret_cast<const float4*>(crow + half + i0 + 4);
      const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = cv[e];
        sg[e] = first ? -sv[e] : sv[e];
      }
    }
    // |c|, |s| <= 2^30 keep the rotation's products in fp32's range; |s| = 0
    // or >= 2^-30 keeps yp * s (>= 2^-90) where its fma error term is exact.
#pragma unroll
    for (int e = 0; e < 8; ++e)
      cs_ok = cs_ok && fabsf(c[e]) <= 0x1p30f && fabsf(sg[e]) <= 0x1p30f &&
              (sg[e] == 0.0f || fabsf(sg[e]) >= 0x1p-30f);
  }
  if (!p.interleaved && rot > 0) {
    const int half = rot / 2, hs = half / 8;
    if (d0 < half) src = lane + hs;
    else if (d0 < rot) src = lane - hs;
  }

  const int H = p.Hq + p.Hkv;
  uint16_t* qrow = p.q + b * p.q_sb + s * p.q_ss + d0;
  uint16_t* krow = p.k + b * p.k_sb + s * p.k_ss + d0 - static_cast<int64_t>(p.Hq) * p.k_sh;
  const double eps = static_cast<double>(p.eps);
  auto row_ptr = [&](int h) { return h < p.Hq ? qrow + h * p.q_sh : krow + h * p.k_sh; };

  uint4 xv[BATCH];
#pragma unroll
  for (int j = 0; j < BATCH; ++j)
    xv[j] = (valid && j < H) ? *reinterpret_cast<const uint4*>(row_ptr(j)) : make_uint4(0, 0, 0, 0);

  for (int h0 = 0; h0 < H; h0 += BATCH) {
    // next batch in flight while this one computes
    uint4 xn[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int h = h0 + BATCH + j;
      xn[j] = (valid && h < H) ? *reinterpret_cast<const uint4*>(row_ptr(h)) : make_uint4(0, 0, 0, 0);
    }
    // sums of squares in fp64 (the bf16 -> fp64 conversions are exact)
    double ss[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const uint32_t xw[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
      ss[j] = 0.0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const double a = static_cast<double>(bf16_lo(xw[i]));
        const double a2 = static_cast<double>(bf16_hi(xw[i]));
        ss[j] += a * a;
        ss[j] += a2 * a2;
      }
    }
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) {
#pragma unroll
      for (int j = 0; j < BATCH; ++j) ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], o);
    }
    // lane j of the group takes row j's square root and division
    double mine = ss[0];
#pragma unroll
    for (int j = 1; j < BATCH; ++j) mine = (sub % BATCH == j) ? ss[j] : mine;
    const double r_mine = 1.0 / sqrt(mine / static_cast<double>(D) + eps);
    const int gbase = lane & ~(TPR - 1);

#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int h = h0 + j;
      const double r = __shfl_sync(0xffffffffu, r_mine, gbase + j);
      if (h >= H) break;
      const bool is_q = h < p.Hq;
      const float* w = w_s[is_q ? 0 : 1] + d0;
      const bool general = valid && (!(r >= 0x1p-100 && r <= 0x1p100) || !cs_ok || !(is_q ? wq_ok : wk_ok));
      uint4 o;
      if (__any_sync(0xffffffffu, general)) {
        o = row_general(xv[j], w, r, c, sg, p.interleaved, src, rotates);
      } else {
        const float r_f = __double2float_rn(r);
        const uint32_t xw[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
        const float4 w0 = *reinterpret_cast<const float4*>(w);
        const float4 w1 = *reinterpret_cast<const float4*>(w + 4);
        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        bool fix = false;
        uint32_t yb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float ya = norm_fp32(bf16_lo(xw[i]), r_f, wv[2 * i], fix);
          const float yc = norm_fp32(bf16_hi(xw[i]), r_f, wv[2 * i + 1], fix);
          yb[i] = pack_bf16x2_rn(ya, yc);
        }
        if (fix) {  // exact y for this lane's 8 dims
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t lo = bf16_bits_rn(bf16_to_f64(xw[i] & 0xFFFFu) * r * static_cast<double>(wv[2 * i]));
            const uint32_t hi = bf16_bits_rn(bf16_to_f64(xw[i] >> 16) * r * static_cast<double>(wv[2 * i + 1]));
            yb[i] = lo | (hi << 16);
          }
        }
        uint32_t pb[4];
        if (p.interleaved) {
#pragma unroll
          for (int i = 0; i < 4; ++i) pb[i] = __byte_perm(yb[i], 0, 0x1032);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) pb[i] = __shfl_sync(0xffffffffu, yb[i], src);
        }
        fix = false;
        uint32_t zb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float za = rot_fp32(bf16_lo(yb[i]), bf16_lo(pb[i]), c[2 * i], sg[2 * i], fix);
          const float zc = rot_fp32(bf16_hi(yb[i]), bf16_hi(pb[i]), c[2 * i + 1], sg[2 * i + 1], fix);
          zb[i] = pack_bf16x2_rn(za, zc);
        }
        if (fix) {  // exact rotation for this lane's 8 dims
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t lo = bf16_bits_rn(fma(static_cast<double>(bf16_lo(pb[i])), static_cast<double>(sg[2 * i]),
                                                 static_cast<double>(bf16_lo(yb[i])) * static_cast<double>(c[2 * i])));
            const uint32_t hi = bf16_bits_rn(fma(static_cast<double>(bf16_hi(pb[i])), static_cast<double>(sg[2 * i + 1]),
                                                 static_cast<double>(bf16_hi(yb[i])) * static_cast<double>(c[2 * i + 1])));
            zb[i] = lo | (hi << 16);
          }
        }
        if (!rotates) {  // past rot_dim: y itself
#pragma unroll
          for (int i = 0; i < 4; ++i) zb[i] = yb[i];
        }
        o = make_uint4(zb[0], zb[1], zb[2], zb[3]);
      }
      if (valid) *reinterpret_cast<uint4*>(row_ptr(h)) = o;
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) xv[j] = xn[j];
  }
}

constexpr int kFastThreads = 256;

// 16-byte store with the streaming (evict-first) cache hint: the rewritten
// rows are not read again by this kernel, so their L2 lines go first.
__device__ __forceinline__ void st_stream_v4(uint16_t* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// fp32 instance, one token per warp: 32 / (D/8) rows per load instruction,
// so a warp streams through its token's heads in contiguous runs (BATCH
// loads of (32 / (D/8)) consecutive heads per iteration, the next batch in
// flight).  One block per kFastThreads / 32 tokens, MINB blocks per SM: the
// bytes in flight per SM are set by the warps resident and BATCH.
template <int D, int BATCH, int MINB>
__global__ void __launch_bounds__(kFastThreads, MINB) qk_norm_rope_warp_kernel(const NormRopeParams p) {
  constexpr int TPR = D / 8;            // lanes per row
  constexpr int RPW = 32 / TPR;         // rows per warp-wide load
  constexpr int STEP = RPW * BATCH;     // heads per iteration
  __shared__ __align__(16) float w_s[2][D];
  for (int i = threadIdx.x; i < 2 * D; i += blockDim.x)
    w_s[i / D][i % D] = __uint_as_float(static_cast<uint32_t>((i < D ? p.w_q : p.w_k)[i % D]) << 16);
  __syncthreads();

  const int lane = threadIdx.x % 32;
  const int sub = lane % TPR;
  const int g = lane / TPR;             // row within a warp-wide load
  const int d0 = sub * 8;
  const int rot = p.rot_dim;
  const bool rotates = d0 < rot;
  int src = lane;
  if (!p.interleaved && rot > 0) {
    const int half = rot / 2, hs = half / 8;
    if (d0 < half) src = lane + hs;
    else if (d0 < rot) src = lane - hs;
  }
  const int H = p.Hq + p.Hkv;
  const float inv_d = 1.0f / static_cast<float>(D);
  const int64_t n_tok = static_cast<int64_t>(p.B) * p.S;
  const int64_t tok = static_cast<int64_t>(blockIdx.x) * (kFastThreads / 32) + threadIdx.x / 32;
  if (tok >= n_tok) return;  // whole warps: every shuffle below has all 32 lanes
  const int s = static_cast<int>(tok % p.S);
  const int b = static_cast<int>(tok / p.S);
  float c[8], sg[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) { c[i] = 1.0f; sg[i] = 0.0f; }
  if (rotates) {
    const float* crow = p.table + static_cast<int64_t>(s) * rot;
    if (p.interleaved) {
      const float4 c4 = *reinterpret_cast<const float4*>(crow + d0 / 2);
      const float4 s4 = *reinterpret_cast<const float4*>(crow + rot / 2 + d0 / 2);
      const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
      const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        c[2 * e] = c[2 * e + 1] = cv[e];
        sg[2 * e] = -sv[e];
        sg[2 * e + 1] = sv[e];
      }
    } else {
      const int half = rot / 2;
      const bool first = d0 < half;
      const int i0 = first ? d0 : d0 - half;
      const float4 c0 = *reinterpret_cast<const float4*>(crow + i0);
      const float4 c1 = *reinterpret_cast<const float4*>(crow + i0 + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(crow + half + i0);
      const float4 s1 = *reinterpret_cast<const float4*>(crow + half + i0 + 4);
      const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = cv[e];
        sg[e] = first ? -sv[e] : sv[e];
      }
    }
  }
  uint16_t* qrow = p.q + b * p.q_sb + s * p.q_ss + d0;
  uint16_t* krow = p.k + b * p.k_sb + s * p.k_ss + d0 - static_cast<int64_t>(p.Hq) * p.k_sh;
  auto row_ptr = [&](int h) { return h < p.Hq ? qrow + h * p.q_sh : krow + h * p.k_sh; };

  uint4 xv[BATCH];
#pragma unroll
  for (int j = 0; j < BATCH; ++j) {
    const int h = g + RPW * j;
    xv[j] = h < H ? *reinterpret_cast<const uint4*>(row_ptr(h)) : make_uint4(0, 0, 0, 0);
  }
  for (int h0 = 0; h0 < H; h0 += STEP) {
    uint4 xn[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int h = h0 + STEP + g + RPW * j;
      xn[j] = h < H ? *reinterpret_cast<const uint4*>(row_ptr(h)) : make_uint4(0, 0, 0, 0);
    }
    float ss[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const uint32_t xw[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
      float a = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = bf16_lo(xw[i]), hi = bf16_hi(xw[i]);
        a = fmaf(lo, lo, a);
        a = fmaf(hi, hi, a);
      }
      ss[j] = a;
    }
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) {
#pragma unroll
      for (int j = 0; j < BATCH; ++j) ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], o);
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int h = h0 + g + RPW * j;
      const float r = rsqrtf(fmaf(ss[j], inv_d, p.eps));
      const float* w = w_s[h < p.Hq ? 0 : 1] + d0;
      const float4 w0 = *reinterpret_cast<const float4*>(w);
      const float4 w1 = *reinterpret_cast<const float4*>(w + 4);
      const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      const uint32_t xw[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
      uint32_t yb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        yb[i] = pack_bf16x2_rn(bf16_lo(xw[i]) * r * wv[2 * i], bf16_hi(xw[i]) * r * wv[2 * i + 1]);
      uint32_t pb[4];
      if (p.interleaved) {
#pragma unroll
        for (int i = 0; i < 4; ++i) pb[i] = __byte_perm(yb[i], 0, 0x1032);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) pb[i] = __shfl_sync(0xffffffffu, yb[i], src);
      }
      uint32_t zb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float za = fmaf(bf16_lo(pb[i]), sg[2 * i], bf16_lo(yb[i]) * c[2 * i]);
        const float zc = fmaf(bf16_hi(pb[i]), sg[2 * i + 1], bf16_hi(yb[i]) * c[2 * i + 1]);
        zb[i] = rotates ? pack_bf16x2_rn(za, zc) : yb[i];
      }
      if (h < H) st_stream_v4(row_ptr(h), make_uint4(zb[0], zb[1], zb[2], zb[3]));
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) xv[j] = xn[j];
  }
}


inline cudaError_t launch(const NormRopeParams& p, int D, bool exact, cudaStream_t stream) {
  const int64_t tokens = static_cast<int64_t>(p.B) * p.S;
  const int groups = kNormRopeThreads / (D / 8);
  const int64_t blocks = (tokens + groups - 1) / groups;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  if (blocks == 0) return cudaSuccess;
  const unsigned g = static_cast<unsigned>(blocks);
  if (exact) {
    switch (D) {
      case 64: qk_norm_rope_kernel<64><<<g, kNormRopeThreads, 0, stream>>>(p); break;
      case 128: qk_norm_rope_kernel<128><<<g, kNormRopeThreads, 0, stream>>>(p); break;
      case 256: qk_norm_rope_kernel<256><<<g, kNormRopeThreads, 0, stream>>>(p); break;
      default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
  }
  // one token per warp, kFastThreads / 32 tokens per block, 4 blocks per SM
  const int64_t wblocks = (tokens + kFastThreads / 32 - 1) / (kFastThreads / 32);
  if (wblocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  const unsigned gw = static_cast<unsigned>(wblocks);
  switch (D) {
    case 64: qk_norm_rope_warp_kernel<64, 2, 4><<<gw, kFastThreads, 0, stream>>>(p); break;
    case 128: qk_norm_rope_warp_kernel<128, 2, 4><<<gw, kFastThreads, 0, stream>>>(p); break;
    case 256: qk_norm_rope_warp_kernel<256, 2, 4><<<gw, kFastThreads, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace skqkn
