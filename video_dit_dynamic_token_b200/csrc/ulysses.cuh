// Light-Ulysses exchange kernels: FP8 row quantisation and the layout changes
// around the sequence <-> head all-to-all.
//
// "600倍加速，720p视频实时生成！单卡也能带的动14B模型", §多卡路径: Ulysses
// sequence parallelism moves the data between the sequence and head
// dimensions with an all-to-all; the exchanged data is FP8 and Q, K, V travel
// as one payload.  This library's reading of the rest: rank r holds tokens
// [r Lr, (r+1) Lr) of every head before the exchange and heads [r Hr, (r+1) Hr)
// of all tokens after it; one FP8 scale per (token, head, tensor) row of D
// values, s = absmax/448 (1 for an all-zero row), code = E4M3_rn_satfinite(
// fl32(x * fl32(448/absmax))); the receiver takes bf16(fl32(decode * s)).
//
// One payload buffer per exchange, one segment of `seg` bytes per destination
// rank n (so that a single all-to-all with equal splits moves it):
//   Q/K/V segment: codes [B][Hc][Lr][3][D] uint8, then at byte offset sc_off
//                  scales [B][Hc][Lr][3] fp32
//   output segment: codes [B][Hc][Lr][D], then scales [B][Hc][Lr]
// where Hc is the number of heads of one exchange (a chunk of the Hr heads of
// each destination, starting at head h0 of its range); sc_off and seg are the
// code and scale byte counts rounded up to 16.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "quant.cuh"

namespace lx {

struct BhldRW {  // bf16 [B,H,L,D] view with element strides, readable or writable
  __nv_bfloat16* p;
  long long sB, sH, sL;
};

enum UlyssesMode : int { kPackQKV = 0, kPackO = 1, kUnpackQKV = 2, kUnpackO = 3 };

struct UlyssesArgs {
  BhldRW x[3];      // pack QKV: q, k, v shards [B, H, Lr, D]; unpack QKV: q, k, v chunks [B, Hc, L, D];
                    // pack O: o chunk [B, Hc, L, D]; unpack O: out shard [B, H, Lr, D]
  uint8_t* payload;
  long long seg;     // bytes per destination segment
  long long sc_off;  // byte offset of the scales within a segment
  int N, B, Hr, Hc, h0, Lr;
  long long rows;    // rows of the payload (all segments)
};

// Four consecutive E4M3 codes (lowest byte first) to floats.
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t c, float (&f)[4]) {
  uint32_t lo, hi;
  asm("{\n .reg .b16 a, b;\n mov.b32 {a, b}, %2;\n cvt.rn.f16x2.e4m3x2 %0, a;\n cvt.rn.f16x2.e4m3x2 %1, b;\n}"
      : "=r"(lo), "=r"(hi)
      : "r"(c));
  const __half2 h0 = *reinterpret_cast<const __half2*>(&lo), h1 = *reinterpret_cast<const __half2*>(&hi);
  f[0] = __low2float(h0);
  f[1] = __high2float(h0);
  f[2] = __low2float(h1);
  f[3] = __high2float(h1);
}

// One payload row per D/8 consecutive lanes (16 bytes of bf16 or 8 bytes of
// codes each).  blockIdx.y is the (destination n, batch b, head j) slice of the
// payload, decoded once per CTA; blockIdx.x walks the slice's Lr*X rows (X = 3
// for the Q/K/V payload: row = 3 t + tensor), kUlyPasses groups per lane group,
// with every pass's loads issued before any of them is used.
constexpr int kUlyPasses = 4;

template <int D, int MODE>
__global__ void __launch_bounds__(256) ulysses_rows_kernel(UlyssesArgs a) {
  constexpr int CH = D / 8;
  constexpr int G = 256 / CH;  // row groups per pass
  constexpr bool QKV = MODE == kPackQKV || MODE == kUnpackQKV;
  constexpr int X = QKV ? 3 : 1;
  const int c = threadIdx.x % CH, g = threadIdx.x / CH;
  const int ny = blockIdx.y;
  const int j = ny % a.Hc;
  const int b = (ny / a.Hc) % a.B;
  const int n = ny / (a.Hc * a.B);
  const int slice_rows = a.Lr * X;
  // the slice's first row within destination n's segment
  const long long slice0 = (long long)(ny - n * a.B * a.Hc) * slice_rows;
  uint8_t* codes = a.payload + (long long)n * a.seg;
  float* scales = reinterpret_cast<float*>(codes + a.sc_off);
  const int base = blockIdx.x * G * kUlyPasses;
  __nv_bfloat16* xr[kUlyPasses];
  long long pr[kUlyPasses];
  bool live[kUlyPasses];
#pragma unroll
  for (int i = 0; i < kUlyPasses; ++i) {
    const int lr = base + i * G + g;
    live[i] = lr < slice_rows;
    const int l = live[i] ? lr : 0;
    const int x = QKV ? l % 3 : 0;
    const int t = QKV ? l / 3 : l;
    const BhldRW& T = a.x[x];
    long long head, tok;
    if (MODE == kPackQKV || MODE == kUnpackO) {  // sequence shard, all heads
      head = (long long)n * a.Hr + a.h0 + j;
      tok = t;
    } else {                                      // head chunk, all tokens
      head = j;
      tok = (long long)n * a.Lr + t;
    }
    xr[i] = T.p + b * T.sB + head * T.sH + tok * T.sL + c * 8;
    pr[i] = slice0 + l;
  }
  if constexpr (MODE == kPackQKV || MODE == kPackO) {
    uint4 v[kUlyPasses];
#pragma unroll
    for (int i = 0; i < kUlyPasses; ++i) v[i] = live[i] ? ld_stream_v4(xr[i]) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < kUlyPasses; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      // |x| maxima on bf16 pairs (exact), then over the row's lanes
      __nv_bfloat162 m2 = __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[0]));
#pragma unroll
      for (int e = 1; e < 4; ++e) m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[e])));
      float m = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
      for (int off = 1; off < CH; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      const float inv = m > 0.f ? __fdiv_rn(448.0f, m) : 0.f;
      // fl32(x * inv) in packed pairs (one rounding each, as __fmul_rn)
      const uint64_t inv2 = f2pack(inv, inv);
      float y[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) f2unpack(mul2(f2pack(bf16lo(w[e]), bf16hi(w[e])), inv2), y[2 * e], y[2 * e + 1]);
      const uint32_t c0 = e4m3x4(y[0], y[1], y[2], y[3]);
      const uint32_t c1 = e4m3x4(y[4], y[5], y[6], y[7]);
      if (live[i]) {
        *reinterpret_cast<uint2*>(codes + pr[i] * D + c * 8) = make_uint2(c0, c1);
        if (c == 0) scales[pr[i]] = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
      }
    }
  } else {
    uint2 cw[kUlyPasses];
    float s[kUlyPasses];
#pragma unroll
    for (int i = 0; i < kUlyPasses; ++i) {
      cw[i] = live[i] ? *reinterpret_cast<const uint2*>(codes + pr[i] * D + c * 8) : make_uint2(0, 0);
      s[i] = live[i] ? scales[pr[i]] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kUlyPasses; ++i) {
      if (!live[i]) continue;
      float f0[4], f1[4];
      e4m3x4_to_f32(cw[i].x, f0);
      e4m3x4_to_f32(cw[i].y, f1);
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        __nv_bfloat162 p0 = __floats2bfloat162_rn(__fmul_rn(f0[2 * e], s[i]), __fmul_rn(f0[2 * e + 1], s[i]));
        __nv_bfloat162 p1 = __floats2bfloat162_rn(__fmul_rn(f1[2 * e], s[i]), __fmul_rn(f1[2 * e + 1], s[i]));
        o[e] = *reinterpret_cast<uint32_t*>(&p0);
        o[2 + e] = *reinterpret_cast<uint32_t*>(&p1);
      }
      *reinterpret_cast<uint4*>(xr[i]) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace lx
