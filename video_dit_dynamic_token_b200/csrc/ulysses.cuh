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
// Buffers (dense, row-major):
//   Q/K/V payload to rank n: codes [N][B][Hc][Lr][3][D], scales [N][B][Hc][Lr][3]
//   output payload to rank n: codes [N][B][Hc][Lr][D],   scales [N][B][Hc][Lr]
// where Hc is the number of heads of one exchange (a chunk of the Hr heads of
// each destination, starting at head h0 of its range).
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
  uint8_t* codes;
  float* scales;
  int N, B, Hr, Hc, h0, Lr;
  long long rows;   // rows of the payload
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
// codes each), in payload order.
template <int D, int MODE>
__global__ void __launch_bounds__(256) ulysses_rows_kernel(UlyssesArgs a) {
  constexpr int CH = D / 8;
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / CH;
  const int c = threadIdx.x % CH;
  const bool live = row < a.rows;
  const long long rr = live ? row : 0;
  // payload coordinates of the row
  constexpr bool QKV = MODE == kPackQKV || MODE == kUnpackQKV;
  long long q = rr;
  int x = 0;
  if (QKV) {
    x = (int)(q % 3);
    q /= 3;
  }
  const int t = (int)(q % a.Lr);
  q /= a.Lr;
  const int j = (int)(q % a.Hc);
  q /= a.Hc;
  const int b = (int)(q % a.B);
  const int n = (int)(q / a.B);
  // the bf16 row this payload row comes from or goes to
  const BhldRW& X = a.x[QKV ? x : 0];
  long long head, tok;
  if (MODE == kPackQKV || MODE == kUnpackO) {  // sequence shard, all heads
    head = (long long)n * a.Hr + a.h0 + j;
    tok = t;
  } else {                                      // head chunk, all tokens
    head = j;
    tok = (long long)n * a.Lr + t;
  }
  __nv_bfloat16* xrow = X.p + b * X.sB + head * X.sH + tok * X.sL + c * 8;
  uint8_t* crow = a.codes + rr * D + c * 8;
  if constexpr (MODE == kPackQKV || MODE == kPackO) {
    const uint4 v = live ? ld_stream_v4(xrow) : make_uint4(0, 0, 0, 0);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf16lo(w[e])), fabsf(bf16hi(w[e]))));
#pragma unroll
    for (int off = 1; off < CH; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float inv = m > 0.f ? __fdiv_rn(448.0f, m) : 0.f;
    const uint32_t c0 = e4m3x4(__fmul_rn(bf16lo(w[0]), inv), __fmul_rn(bf16hi(w[0]), inv),
                               __fmul_rn(bf16lo(w[1]), inv), __fmul_rn(bf16hi(w[1]), inv));
    const uint32_t c1 = e4m3x4(__fmul_rn(bf16lo(w[2]), inv), __fmul_rn(bf16hi(w[2]), inv),
                               __fmul_rn(bf16lo(w[3]), inv), __fmul_rn(bf16hi(w[3]), inv));
    if (live) {
      *reinterpret_cast<uint2*>(crow) = make_uint2(c0, c1);
      if (c == 0) a.scales[rr] = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
    }
  } else {
    if (live) {
      const uint2 cw = *reinterpret_cast<const uint2*>(crow);
      const float s = a.scales[rr];
      float f0[4], f1[4];
      e4m3x4_to_f32(cw.x, f0);
      e4m3x4_to_f32(cw.y, f1);
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        __nv_bfloat162 p0 = __floats2bfloat162_rn(__fmul_rn(f0[2 * e], s), __fmul_rn(f0[2 * e + 1], s));
        __nv_bfloat162 p1 = __floats2bfloat162_rn(__fmul_rn(f1[2 * e], s), __fmul_rn(f1[2 * e + 1], s));
        o[e] = *reinterpret_cast<uint32_t*>(&p0);
        o[2 + e] = *reinterpret_cast<uint32_t*>(&p1);
      }
      *reinterpret_cast<uint4*>(xrow) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace lx
