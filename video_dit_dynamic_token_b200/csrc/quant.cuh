// Quantisers (step a3): Q and K to INT8 with one symmetric scale per
// (b, h, 64-token block); V to FP8 E4M3 with one scale per (b, h, channel).
//
// "600倍加速，720p视频实时生成！单卡也能带的动14B模型", §高效推理算子: the sparse
// attention runs with Q/K in INT8 and V in FP8.  The scale granularity is this
// library's reading: absmax/127 per block for Q/K, absmax/448 per channel for V,
// codes rint(x*(127/a)) clamped to +-127 and E4M3_rn_satfinite(v*(448/a)); both
// code decisions are taken in fp32 with correctly rounded divide and multiply.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "planner.cuh"

namespace lx {

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Bits of fl32(x * inv) + 1.5 * 2^23.  With |x| <= a and inv = fl32(127 / a),
// |fl32(x * inv)| <= 127 (1 + 2^-24), so the sum lies in [2^23, 2^24) where
// the float spacing is 1: the add rounds x * inv to the nearest integer, half
// to even, and the low byte of the bits is that integer as a two's-complement
// int8 in [-127, 127] (the +-127 clamp cannot bind).
__device__ __forceinline__ uint32_t i8_code_bits(float x, float inv) {
  return __float_as_uint(__fadd_rn(__fmul_rn(x, inv), 12582912.0f));
}
// Low bytes of a, b, c, d packed into one word, a in the lowest byte.
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}
// The INT8 codes of the 8 bf16 values of one 16-byte chunk.
__device__ __forceinline__ uint2 i8_codes_x8(const uint4& v, float inv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t t[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    t[2 * e] = i8_code_bits(bf16lo(w[e]), inv);
    t[2 * e + 1] = i8_code_bits(bf16hi(w[e]), inv);
  }
  return make_uint2(pack_low_bytes(t[0], t[1], t[2], t[3]), pack_low_bytes(t[4], t[5], t[6], t[7]));
}

// Two fp32 values to two E4M3 codes (lo in bits 0..7), round to nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r;
}
// four floats to four E4M3 bytes, a in the lowest byte
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n .reg .b16 lo, hi;\n cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n"
      " cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n mov.b32 %0, {lo, hi};\n}"
      : "=r"(r) : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

// ---------------------------------------------------------------------------
// Prologue parameters of the Q/K block pass (per-head RMSNorm and 3D RoPE,
// "600倍加速…", §高效推理算子, last paragraph: 3D RoPE and RMSNorm as fused
// kernels; the formulas are this library's reading):
//   y = rope(x / sqrt(mean_c x_c^2 + eps) * w[h, c]).
// The head dimension is split into the t, h and w parts (dt2, dh2, dw2 channel
// pairs, in that order); pair i of a part turns by pos * theta^(-2i/m), whose
// (cos, sin) sit in `table` at part base + pos * pairs + i.  The token at raster
// index n of the (T, Hh, W) grid has (t, h, w) = (n / (Hh W), (n / W) mod Hh,
// n mod W).  yq / yk receive bf16(y) when their pointer is not null.
struct BhldOut {  // bf16 [B,H,L,D] output with element strides
  __nv_bfloat16* p;
  long long sB, sH, sL;
};
struct ProParams {
  const float* wq;     // [H, D]
  const float* wk;     // [H, D]
  const float2* table; // (cos, sin) per (part, position, pair)
  BhldOut yq, yk;
  float eps;
  int Hh, W;
  int dt2, dh2;        // channel pairs of the t and h parts (the w part has D/2 - dt2 - dh2)
  int offh, offw;      // table offsets of the h and w parts (entries)
};

// ---------------------------------------------------------------------------
// Q/K block pass (steps a1 and a3 in one read): one 128-thread CTA per
// (tensor, b*h, 64-token block).  The D/8 16-byte chunks of a row go to
// consecutive lanes (a warp loads whole rows, coalesced) and the 128/(D/8) row
// groups of the CTA take rows r, r + RG, ...; every thread keeps its D/16 rows
// of one chunk in registers.  MEANS: per-channel sums over the thread's rows,
// then over the row groups in a fixed order (shuffles inside a warp, then the
// four warps in shared memory), divided by the valid token count.  CODES: the
// block absmax (max is exact in any order) gives inv = 127/a, and each value
// becomes rint(x * inv) clamped to +-127; the scale a/127 (1 for an all-zero
// block) is stored per block.  Either part may be switched off, so the pool,
// the quantiser and the fused pass share one code path and agree bit for bit.
// PRO: each valid row is first replaced by the bf16 prologue output (above),
// so the means and codes are those of that bf16 tensor.
// SMOOTH (K smoothing, a variant not on the pages): K's codes are those of
// fl32(k - km[b, h, c]) over the block's valid rows, km the channel means of K.
template <int D, bool MEANS, bool CODES, bool PRO, bool SMOOTH = false>
__global__ void __launch_bounds__(128) qk_block_pass_kernel(BhldView q, BhldView k, float* __restrict__ mq,
                                                           float* __restrict__ mk, int8_t* __restrict__ qc,
                                                           int8_t* __restrict__ kc, float* __restrict__ qs,
                                                           float* __restrict__ ks, int H, int L, int nB,
                                                           ProParams pro, const float* __restrict__ km = nullptr) {
  constexpr int CH = D / 8;      // 16-byte chunks per row
  constexpr int RG = 128 / CH;   // row groups in the CTA
  constexpr int NR = kBlock / RG;  // rows per thread (= D/16)
  const BhldView X = blockIdx.y == 0 ? q : k;
  const long long unit = blockIdx.x;
  const long long bh = unit / nB;
  const int blk = (int)(unit - bh * nB);
  const long long b = bh / H, h = bh - b * H;
  const int t0 = blk * kBlock;
  const int cnt = min(kBlock, L - t0);
  const int c = threadIdx.x % CH, r = threadIdx.x / CH;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const __nv_bfloat16* src = X.p + b * X.sB + h * X.sH + (long long)(t0 + r) * X.sL + c * 8;
  uint4 v[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) v[i] = r + RG * i < cnt ? ld_stream_v4(src + (long long)(RG * i) * X.sL) : make_uint4(0, 0, 0, 0);
  if constexpr (PRO) {
    const bool isk = blockIdx.y != 0;
    // this thread's 8 channels: weights and, for each of its 4 pairs, the
    // table part (0 t, 1 h, 2 w), base and pairs per position
    const float4* wrow = reinterpret_cast<const float4*>((isk ? pro.wk : pro.wq) + h * D + c * 8);
    const float4 w0 = __ldg(wrow), w1 = __ldg(wrow + 1);
    // weights of this thread's 4 channel pairs, packed for f32x2 arithmetic
    const uint64_t wp[4] = {f2pack(w0.x, w0.y), f2pack(w0.z, w0.w), f2pack(w1.x, w1.y), f2pack(w1.z, w1.w)};
    int pax[4], pbase[4], pstride[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int pi = 4 * c + j;
      if (pi < pro.dt2) {
        pax[j] = 0; pbase[j] = pi; pstride[j] = pro.dt2;
      } else if (pi < pro.dt2 + pro.dh2) {
        pax[j] = 1; pbase[j] = pro.offh + (pi - pro.dt2); pstride[j] = pro.dh2;
      } else {
        pax[j] = 2; pbase[j] = pro.offw + (pi - pro.dt2 - pro.dh2); pstride[j] = D / 2 - pro.dt2 - pro.dh2;
      }
    }
    const BhldOut Y = isk ? pro.yk : pro.yq;
    // grid position of this thread's first row; the later rows (RG apart) are
    // reached by adding to w and carrying into h and t
    int pt, ph, pw;
    {
      const int n = t0 + r;
      const int nw = n / pro.W;
      pw = n - nw * pro.W;
      pt = nw / pro.Hh;
      ph = nw - pt * pro.Hh;
    }
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      if (i > 0) {
        pw += RG;
        while (pw >= pro.W) {
          pw -= pro.W;
          if (++ph == pro.Hh) {
            ph = 0;
            ++pt;
          }
        }
      }
      const int row = r + RG * i;
      // the row's 8 channels as 4 packed (even, odd) pairs
      const uint32_t wd[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint64_t x2[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) x2[j] = f2pack(bf16lo(wd[j]), bf16hi(wd[j]));
      uint64_t ss2 = mul2(x2[0], x2[0]);
#pragma unroll
      for (int j = 1; j < 4; ++j) ss2 = fma2(x2[j], x2[j], ss2);
      float s0, s1;
      f2unpack(ss2, s0, s1);
      float ss = s0 + s1;
      // the row's D/8 chunks sit in consecutive lanes: fold them (every lane
      // takes part, rows past L included, whose values are zero)
#pragma unroll
      for (int off = 1; off < CH; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (row < cnt) {
        const float inv = rsqrtf(ss * (1.0f / (float)D) + pro.eps);  // within 2 fp32 ulps
        const uint64_t inv2 = f2pack(inv, inv);
        const int n = t0 + row;
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int pos = pax[j] == 0 ? pt : (pax[j] == 1 ? ph : pw);
          const float2 cs = __ldg(pro.table + pbase[j] + pos * pstride[j]);
          // u = x * w per channel; (y0, y1) = inv * (ua cos - ub sin, ua sin + ub cos)
          float ua, ub;
          f2unpack(mul2(x2[j], wp[j]), ua, ub);
          const uint64_t p2 = mul2(f2pack(ub, ub), f2pack(-cs.y, cs.x));
          const uint64_t y2 = mul2(fma2(f2pack(ua, ua), f2pack(cs.x, cs.y), p2), inv2);
          float y0, y1;
          f2unpack(y2, y0, y1);
          __nv_bfloat162 yb = __floats2bfloat162_rn(y0, y1);
          o[j] = *reinterpret_cast<uint32_t*>(&yb);
        }
        v[i] = make_uint4(o[0], o[1], o[2], o[3]);
        if (Y.p) *reinterpret_cast<uint4*>(Y.p + b * Y.sB + h * Y.sH + (long long)n * Y.sL + c * 8) = v[i];
      }
    }
  }
  __shared__ float part[MEANS ? 4 : 1][MEANS ? D : 1];
  __shared__ float red[4];
  if constexpr (MEANS) {
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < NR; ++i) acc_bf16x8(a, v[i]);
#pragma unroll
    for (int off = CH; off < 32; off <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) a[e] += __shfl_xor_sync(0xffffffffu, a[e], off);
    if (lane < CH)
#pragma unroll
      for (int e = 0; e < 8; ++e) part[warp][c * 8 + e] = a[e];
  }
  float amax = 0.f;
  const bool smooth = SMOOTH && blockIdx.y != 0;
  float kmv[8];
  if constexpr (SMOOTH) {
#pragma unroll
    for (int e = 0; e < 8; ++e) kmv[e] = 0.f;
    if (smooth) {
      const float4* kmr = reinterpret_cast<const float4*>(km + bh * D + c * 8);
      const float4 a0 = __ldg(kmr), a1 = __ldg(kmr + 1);
      kmv[0] = a0.x; kmv[1] = a0.y; kmv[2] = a0.z; kmv[3] = a0.w;
      kmv[4] = a1.x; kmv[5] = a1.y; kmv[6] = a1.z; kmv[7] = a1.w;
    }
  }
  if constexpr (CODES) {
    if (smooth) {
      // |k - km| over the valid rows (the zero-filled rows past L would count |km|)
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        if (r + RG * i < cnt) {
          const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            amax = fmaxf(amax, fabsf(bf16lo(w[e]) - kmv[2 * e]));
            amax = fmaxf(amax, fabsf(bf16hi(w[e]) - kmv[2 * e + 1]));
          }
        }
      }
    } else {
      // |x| maxima on bf16 pairs (exact: widening to fp32 keeps order, and both
      // maxima ignore a NaN operand as fmaxf does)
      __nv_bfloat162 m2 = __floats2bfloat162_rn(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[e])));
      }
      amax = fmaxf(__low2float(m2), __high2float(m2));
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) red[warp] = amax;
  }
  __syncthreads();
  if constexpr (MEANS) {
    if (threadIdx.x < D) {
      const float sum = ((part[0][threadIdx.x] + part[1][threadIdx.x]) + part[2][threadIdx.x]) + part[3][threadIdx.x];
      float* __restrict__ M = blockIdx.y == 0 ? mq : mk;
      M[(bh * nB + blk) * D + threadIdx.x] = __fdiv_rn(sum, (float)cnt);
    }
  }
  if constexpr (CODES) {
    amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float inv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
    int8_t* __restrict__ C = blockIdx.y == 0 ? qc : kc;
    int8_t* dst = C + (bh * L + t0 + r) * D + c * 8;
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      if (r + RG * i < cnt) {
        uint2 o;
        if (smooth) {
          const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
          uint32_t t8[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            t8[2 * e] = i8_code_bits(bf16lo(w[e]) - kmv[2 * e], inv);
            t8[2 * e + 1] = i8_code_bits(bf16hi(w[e]) - kmv[2 * e + 1], inv);
          }
          o = make_uint2(pack_low_bytes(t8[0], t8[1], t8[2], t8[3]), pack_low_bytes(t8[4], t8[5], t8[6], t8[7]));
        } else {
          o = i8_codes_x8(v[i], inv);
        }
        *reinterpret_cast<uint2*>(dst + (long long)(RG * i) * D) = o;
      }
    }
    if (threadIdx.x == 0) {
      float* __restrict__ S = blockIdx.y == 0 ? qs : ks;
      S[bh * nB + blk] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 1.0f;
    }
  }
}

// ---------------------------------------------------------------------------
// V, pass 1: per-channel absmax.  One 128-thread CTA per (b*h, 512-token span);
// lanes cover 16-byte channel chunks; the CTA folds its rows in shared memory
// and merges into the (zero-initialised) per-channel maxima with atomicMax on
// the bit patterns (non-negative floats order like unsigned ints).
constexpr int kVSpan = 512;
template <int D>
__global__ void __launch_bounds__(128) v_absmax_kernel(BhldView v, uint32_t* __restrict__ amax, int H, int L,
                                                      int nSpan) {
  constexpr int CH = D / 8;        // chunks per row
  constexpr int RPP = 128 / CH;    // rows per pass
  const long long bh = blockIdx.x / nSpan;
  const int span = (int)(blockIdx.x - bh * nSpan);
  const long long b = bh / H, h = bh - b * H;
  const int c = threadIdx.x % CH, r0 = threadIdx.x / CH;
  const int t_begin = span * kVSpan, t_end = min(L, t_begin + kVSpan);
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const __nv_bfloat16* base = v.p + b * v.sB + h * v.sH + c * 8;
  for (int t = t_begin + r0; t < t_end; t += RPP) {
    const uint4 x = ld_stream_v4(base + (long long)t * v.sL);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      m[2 * e] = fmaxf(m[2 * e], fabsf(bf16lo(w[e])));
      m[2 * e + 1] = fmaxf(m[2 * e + 1], fabsf(bf16hi(w[e])));
    }
  }
  __shared__ float red[128][9];
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.x][e] = m[e];
  __syncthreads();
  if (threadIdx.x < D) {
    const int ch = threadIdx.x / 8, e = threadIdx.x % 8;
    float mm = 0.f;
    for (int r = 0; r < RPP; ++r) mm = fmaxf(mm, red[r * CH + ch][e]);
    atomicMax(amax + bh * D + threadIdx.x, __float_as_uint(mm));
  }
}

// ---------------------------------------------------------------------------
// V, pass 2: codes.  A unit is one (b*h, 64-token block); each persistent
// 128-thread CTA walks a contiguous range of units.  As in the Q/K pass, the
// D/8 16-byte chunks of a row go to consecutive lanes and thread t takes rows
// r, r + RG, ... of chunk c = t mod (D/8), so a warp loads and stores whole
// rows; the next unit's rows are loaded into a second register set while the
// current one is converted.  A thread's 8 channels never change, so their
// reciprocal scales live in registers and are rebuilt when b*h changes; the
// CTA that converts block 0 of a head also writes the head's channel scales.
template <int D>
__global__ void __launch_bounds__(128, 4) v_quant_kernel(BhldView v, const uint32_t* __restrict__ amax,
                                                        uint8_t* __restrict__ vc, float* __restrict__ vs, int H,
                                                        int L, int nB, long long nunits, long long units_per_cta) {
  constexpr int CH = D / 8;        // 16-byte chunks per row
  constexpr int RG = 128 / CH;     // row groups in the CTA
  constexpr int NR = kBlock / RG;  // rows per thread
  const long long u_begin = (long long)blockIdx.x * units_per_cta;
  const long long u_end = min(u_begin + units_per_cta, nunits);
  if (u_begin >= u_end) return;
  const int c = threadIdx.x % CH, r = threadIdx.x / CH;
  uint4 x[NR], xn[NR];
  long long bh = u_begin / nB;
  int blk = (int)(u_begin - bh * nB);
  {
    const long long b = bh / H, h = bh - b * H;
    const __nv_bfloat16* src = v.p + b * v.sB + h * v.sH + (long long)(blk * kBlock + r) * v.sL + c * 8;
    const int cnt = min(kBlock, L - blk * kBlock);
#pragma unroll
    for (int i = 0; i < NR; ++i) x[i] = r + RG * i < cnt ? ld_stream_v4(src + (long long)(RG * i) * v.sL) : make_uint4(0, 0, 0, 0);
  }
  long long bh_s = -1;  // head whose scales sit in inv
  float inv[8];
  for (long long u = u_begin; u < u_end; ++u) {
    const long long bhn = (u + 1) / nB;
    const int blkn = (int)(u + 1 - bhn * nB);
    if (u + 1 < u_end) {
      const long long b = bhn / H, h = bhn - b * H;
      const __nv_bfloat16* src = v.p + b * v.sB + h * v.sH + (long long)(blkn * kBlock + r) * v.sL + c * 8;
      const int cnt = min(kBlock, L - blkn * kBlock);
#pragma unroll
      for (int i = 0; i < NR; ++i)
        xn[i] = r + RG * i < cnt ? ld_stream_v4(src + (long long)(RG * i) * v.sL) : make_uint4(0, 0, 0, 0);
    }
    if (bh != bh_s) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float a = __uint_as_float(amax[bh * D + c * 8 + e]);
        inv[e] = a > 0.f ? __fdiv_rn(448.0f, a) : 0.f;
      }
      bh_s = bh;
    }
    if (blk == 0)
      for (int ch = threadIdx.x; ch < D; ch += blockDim.x) {
        const float a = __uint_as_float(amax[bh * D + ch]);
        vs[bh * D + ch] = a > 0.f ? __fdiv_rn(a, 448.0f) : 1.0f;
      }
    const int cnt = min(kBlock, L - blk * kBlock);
    uint8_t* dst = vc + (bh * L + blk * kBlock + r) * D + c * 8;
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      if (r + RG * i < cnt) {
        const uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
        uint32_t p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          p[e] = e4m3x2(__fmul_rn(bf16lo(w[e]), inv[2 * e]), __fmul_rn(bf16hi(w[e]), inv[2 * e + 1]));
        *reinterpret_cast<uint2*>(dst + (long long)(RG * i) * D) = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
      }
    }
#pragma unroll
    for (int i = 0; i < NR; ++i) x[i] = xn[i];
    bh = bhn;
    blk = blkn;
  }
}

// ---------------------------------------------------------------------------
// K channel means for K smoothing (a variant not on the pages), in two
// deterministic passes: one 128-thread CTA per (b*h, 512-token span) sums its
// rows per channel in fp64 (lanes on 16-byte chunks, rows in order, then the
// row groups in order through shared memory); then one thread per (b*h,
// channel) adds the spans in order, divides by L and rounds to fp32 once.
template <int D>
__global__ void __launch_bounds__(128) k_mean_partial_kernel(BhldView k, double* __restrict__ part, int H, int L,
                                                            int nSpan) {
  constexpr int CH = D / 8;
  constexpr int RPP = 128 / CH;
  const long long bh = blockIdx.x / nSpan;
  const int span = (int)(blockIdx.x - bh * nSpan);
  const long long b = bh / H, h = bh - b * H;
  const int c = threadIdx.x % CH, r0 = threadIdx.x / CH;
  const int t_begin = span * kVSpan, t_end = min(L, t_begin + kVSpan);
  double s[8] = {0., 0., 0., 0., 0., 0., 0., 0.};
  const __nv_bfloat16* base = k.p + b * k.sB + h * k.sH + c * 8;
  for (int t = t_begin + r0; t < t_end; t += RPP) {
    const uint4 x = ld_stream_v4(base + (long long)t * k.sL);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s[2 * e] += (double)bf16lo(w[e]);
      s[2 * e + 1] += (double)bf16hi(w[e]);
    }
  }
  __shared__ double red[128][9];
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.x][e] = s[e];
  __syncthreads();
  if (threadIdx.x < D) {
    const int ch = threadIdx.x / 8, e = threadIdx.x % 8;
    double acc = 0.;
    for (int rr = 0; rr < RPP; ++rr) acc += red[rr * CH + ch][e];
    part[((long long)bh * nSpan + span) * D + threadIdx.x] = acc;
  }
}

__global__ void k_mean_final_kernel(const double* __restrict__ part, float* __restrict__ km, long long BH, int D,
                                    int nSpan, int L) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= BH * D) return;
  const long long bh = i / D;
  const int ch = (int)(i - bh * D);
  double acc = 0.;
  for (int sp = 0; sp < nSpan; ++sp) acc += part[(bh * nSpan + sp) * D + ch];
  km[i] = (float)(acc / (double)L);
}

// ---------------------------------------------------------------------------
// 3D RoPE table: entry e of the t part (then the h part, then the w part) is
// (cos, sin) of pos * theta^(-2i/m) for position pos and pair i of a part of m
// channels; the angle and its sine and cosine are taken in fp64 and rounded
// to fp32 once.
__global__ void rope3d_table_kernel(float2* __restrict__ table, int T, int Hh, int W, int dt2, int dh2, int dw2,
                                    double theta) {
  const int nt = T * dt2, nh = Hh * dh2, nw = W * dw2;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < nt + nh + nw; e += gridDim.x * blockDim.x) {
    int pos, i, pairs;
    if (e < nt) {
      pos = e / dt2; i = e - pos * dt2; pairs = dt2;
    } else if (e < nt + nh) {
      pos = (e - nt) / dh2; i = (e - nt) - pos * dh2; pairs = dh2;
    } else {
      pos = (e - nt - nh) / dw2; i = (e - nt - nh) - pos * dw2; pairs = dw2;
    }
    const double ang = (double)pos * pow(theta, -(double)i / (double)pairs);  // -2i/m with m = 2 pairs
    double sn, cs;
    sincos(ang, &sn, &cs);
    table[e] = make_float2((float)cs, (float)sn);
  }
}

}  // namespace lx
