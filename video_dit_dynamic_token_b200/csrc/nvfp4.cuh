// NVFP4 quantisation and the dual-NVFP4 block-scaled GEMM (tcgen05 kind::mxf4nvf4).
//
// "Run Wan2.2-A14B on One RTX 5090: 720p Video in 3.8s", §2 (NVFP4
// quantization-aware training): NVFP4 holds E2M1 values, one E4M3 scale per
// 16 consecutive elements and one FP32 scale per tensor; the linear layers run
// a block-scaled GEMM of NVFP4 activations by NVFP4 weights with FP32
// accumulation, BF16 output and the column bias added in the epilogue.
//
// The scale rule (the pages give the format, not the rule; the usual NVFP4
// recipe, fixed to fp32 operations so that it is reproducible):
//   g = fl32(amax / 2688)  (1 for an all-zero tensor),  ig6 = fl32(1 / fl32(6 g))
//   s = E4M3_rn_satfinite(fl32(amax_block * ig6)),  inv = fl32(1 / fl32(s g))  (0 if s = 0)
//   code = E2M1_rn_satfinite(fl32(x * inv)), negative zero stored as +0.
//
// Layouts (all dense):
//   codes  [R][K/2] bytes, element 2i in the low nibble of byte i;
//   scales tiled for the MMA: for row r, 16-block j (k-step ks = j/4 of 64
//          elements, jj = j%4), tile t = r/128, lane l = r%32, column c = (r%128)/32,
//          byte (t*KS + ks)*512 + l*16 + c*4 + jj, KS = K/64; rows are padded to
//          a multiple of 128 with zero scales.  One 512-byte chunk is what one
//          tcgen05.cp 32x128b.warpx4 moves into TMEM for one k-step of a
//          128-row tile: TMEM lane l, column c holds the four scales of row
//          32c + l, which is where the block-scaled MMA reads them.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "ptx.cuh"
#include "quant.cuh"

namespace lx {

constexpr float kNvGsDiv = 2688.0f;  // largest E4M3 scale (448) times largest E2M1 value (6)

// ---------------------------------------------------------------- element conversions
// Eight fp32 values (scaled) -> eight E2M1 codes in one word, element 0 in the
// lowest nibble; saturating round-to-nearest-even, negative zero made +0.
__device__ __forceinline__ uint32_t e2m1x8(const float (&y)[8]) {
  uint32_t r;
  asm("{\n .reg .b8 b0, b1, b2, b3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
      " mov.b32 %0, {b0, b1, b2, b3};\n}"
      : "=r"(r)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  // keep a nibble's sign bit only where its magnitude is not zero
  const uint32_t nz = ((r & 0x77777777u) + 0x77777777u) & 0x88888888u;
  return r & (0x77777777u | nz);
}

// Value of one E4M3 code (low byte of c).
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  uint32_t h;
  asm("{\n .reg .b16 a;\n cvt.u16.u32 a, %1;\n cvt.rn.f16x2.e4m3x2 %0, a;\n}" : "=r"(h) : "r"(c & 0xFFu));
  return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------- global scale
// amax of a bf16 [R, K] matrix (row stride ld elements, K % 8 == 0) as float
// bits, atomically max-ed into *amax_bits (zeroed by the caller).
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const __nv_bfloat16* __restrict__ x, long long R, int K,
                                                         long long ld, unsigned* amax_bits) {
  const int nv = K / 8;
  uint32_t m = 0;  // two bf16 magnitudes: unsigned compare orders non-negative floats
  for (long long r = blockIdx.x; r < R; r += gridDim.x) {
    const __nv_bfloat16* row = x + r * ld;
    for (int c = threadIdx.x; c < nv; c += blockDim.x) {
      const uint4 v = ld_stream_v4(row + 8 * c);
      m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    }
  }
  uint32_t b = max(m & 0xFFFFu, m >> 16) << 16;
  b = __reduce_max_sync(0xFFFFFFFFu, b);
  if ((threadIdx.x & 31) == 0 && b) atomicMax(amax_bits, b);
}

// *g holds amax bits on entry and the global scale on exit.
__global__ void nvfp4_gscale_kernel(float* g) {
  const float a = __uint_as_float(*reinterpret_cast<const unsigned*>(g));
  *g = a > 0.f ? __fdiv_rn(a, kNvGsDiv) : 1.0f;
}

// ---------------------------------------------------------------- quantiser
// grid (ceil(R/128), ceil(KS/kNvQSteps)), 128 threads: thread = one row of a
// 128-row tile, kNvQSteps k-steps of 64 elements (128 bytes of bf16 read, 32
// bytes of codes and one 4-scale word written per k-step).  Lane l of warp c
// owns TMEM-layout lane l, column c, so the scale words of a warp land 16 bytes
// apart inside the k-step's 512-byte chunk.
constexpr int kNvQSteps = 4;

__global__ void __launch_bounds__(128) nvfp4_quant_kernel(const __nv_bfloat16* __restrict__ x, long long R, int K,
                                                          long long ld, const float* __restrict__ gs,
                                                          uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  const int KS = K / 64;
  const long long r = (long long)blockIdx.x * 128 + threadIdx.x;
  const int l = threadIdx.x & 31, c = threadIdx.x >> 5;
  const float g = *gs;
  const float ig6 = __frcp_rn(__fmul_rn(6.0f, g));
  const bool live = r < R;
  const int ks0 = blockIdx.y * kNvQSteps;
#pragma unroll 1
  for (int i = 0; i < kNvQSteps; ++i) {
    const int ks = ks0 + i;
    if (ks >= KS) break;
    uint32_t* sfw = reinterpret_cast<uint32_t*>(sf + ((long long)blockIdx.x * KS + ks) * 512 + l * 16 + c * 4);
    if (!live) {
      *sfw = 0u;
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + r * ld + (long long)ks * 64);
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = ldg_nc_v4(src + j);
    uint32_t cw[8];
    uint32_t sword = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t w[8] = {v[2 * b].x,     v[2 * b].y,     v[2 * b].z,     v[2 * b].w,
                             v[2 * b + 1].x, v[2 * b + 1].y, v[2 * b + 1].z, v[2 * b + 1].w};
      uint32_t m = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) m = __vmaxu2(m, w[e] & 0x7FFF7FFFu);
      const float amax = __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16);
      const uint32_t s8 = e4m3x2(__fmul_rn(amax, ig6), 0.f) & 0xFFu;
      const float s = e4m3_to_f32(s8);
      const float inv = s > 0.f ? __frcp_rn(__fmul_rn(s, g)) : 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float y[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          y[2 * e] = __fmul_rn(bf16lo(w[4 * h + e]), inv);
          y[2 * e + 1] = __fmul_rn(bf16hi(w[4 * h + e]), inv);
        }
        cw[2 * b + h] = e2m1x8(y);
      }
      sword |= s8 << (8 * b);
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + r * (long long)(K / 2) + (long long)ks * 32);
    dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    *sfw = sword;
  }
}

// ---------------------------------------------------------------- GEMM
// Y[m, n] = bf16(fl32(acc * fl32(gx * gw)) + bias[n]),  acc = sum_k x_k w_k in fp32 (TMEM).
// Persistent: one CTA per SM walks the 128 x 256 output tiles t = blockIdx.x,
// blockIdx.x + gridDim.x, ... (N-tile fastest, so that the CTAs running at one
// time share a few A row blocks and the weights stay in L2).  K runs in stages
// of 256 elements (128 bytes per row), four k-steps of 64 per stage, through a
// ring of kNvStages stages that carries on from one tile to the next, filled by
// TMA (codes, 128-byte swizzle) and plain bulk copies (scales).
//   warp 0, lane 0: loads;
//   warp 1, lane 0: copies each k-step's scales into TMEM (tcgen05.cp), issues
//                   the MMAs and commits the accumulator once per tile;
//   warps 2..9:     drain the accumulator.  Warp w reads TMEM lane quarter w%4
//                   (rows 32(w%4)..+31) and one half of the 256 columns into
//                   registers, hands the accumulator back to the MMA warp at
//                   once, then scales, adds the bias (staged per tile in shared
//                   memory, two buffers) and writes bf16 while the next tile
//                   accumulates.
constexpr int kNvBM = 128, kNvBN = 256, kNvStages = 4;
constexpr int kNvEpiWarps = 8, kNvThreads = 32 * (2 + kNvEpiWarps);  // 320
constexpr uint32_t kNvABytes = 128 * 128;          // A stage: 128 rows x 128 bytes
constexpr uint32_t kNvBBytes = 256 * 128;          // B stage: 256 rows x 128 bytes
constexpr uint32_t kNvSfaBytes = 4 * 512;          // 4 k-steps of one 128-row tile
constexpr uint32_t kNvSfbBytes = 2 * 4 * 512;      // two 128-row tiles
constexpr uint32_t kNvStageBytes = kNvABytes + kNvBBytes + kNvSfaBytes + kNvSfbBytes;  // 55296 = 54 KB
constexpr uint32_t kNvSmemBytes = kNvStages * kNvStageBytes + 1024;                    // + alignment slack
constexpr uint32_t kNvTmemCols = 512;  // accumulator 0..255; scale ring 256 + 48 per stage
// block-scaled instruction descriptor: A, B = E2M1 (1) in [7,10) / [10,13), K-major,
// N >> 3 in [17,23), scale type UE4M3 (bit 23 = 0), M >> 4 in [24,29), scale ids 0
constexpr uint32_t kNvIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kNvBN >> 3) << 17) | ((uint32_t)(kNvBM >> 4) << 24);
static_assert(kNvSmemBytes <= 232448 - 4096, "shared memory per CTA (dynamic + static)");
static_assert(256 + kNvStages * 48 <= (int)kNvTmemCols, "TMEM columns");

struct NvGemmArgs {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* gx;
  const float* gw;
  const float* bias;  // [N] or null
  __nv_bfloat16* y;
  long long ldy;
  int M, N, K;
  unsigned long long limit_ns;
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// 32 TMEM lanes x 128 bits from shared memory, written to all four lane quarters.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                         uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}

// Ties 32 registers written by tcgen05.ld to this point (after tcgen05.wait::ld),
// so that no use of them is scheduled above the wait.
__device__ __forceinline__ void reg_fence32(uint32_t (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(v[i]));
}

// One 32-column chunk of a row: y = bf16(fl32(acc * alpha) + bias).
__device__ __forceinline__ void nv_store_chunk(const uint32_t (&v)[32], const float* sb, float alpha,
                                               __nv_bfloat16* dst) {
  uint32_t o[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 b = reinterpret_cast<const float4*>(sb)[i];
    const float y0 = __fadd_rn(__fmul_rn(__uint_as_float(v[4 * i]), alpha), b.x);
    const float y1 = __fadd_rn(__fmul_rn(__uint_as_float(v[4 * i + 1]), alpha), b.y);
    const float y2 = __fadd_rn(__fmul_rn(__uint_as_float(v[4 * i + 2]), alpha), b.z);
    const float y3 = __fadd_rn(__fmul_rn(__uint_as_float(v[4 * i + 3]), alpha), b.w);
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(y0, y1), p1 = __floats2bfloat162_rn(y2, y3);
    o[2 * i] = *reinterpret_cast<const uint32_t*>(&p0);
    o[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&p1);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) d[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
}

__global__ void __launch_bounds__(kNvThreads, 1) nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                                                                   const __grid_constant__ CUtensorMap tmB,
                                                                   NvGemmArgs a) {
  extern __shared__ uint8_t nv_smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(nv_smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_full[kNvStages], bar_empty[kNvStages], bar_acc_full, bar_acc_empty, bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ int never_abort;
  __shared__ __align__(16) float sbias[2][kNvBN];  // a tile's bias (0 past N or without bias), two buffers

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = a.K / 64, nkb = a.K / 256;
  const int nt128 = (a.N + 127) / 128;  // 128-row tiles of the weight scales
  const int ntn = (a.N + kNvBN - 1) / kNvBN;
  const long long ntiles = (long long)ntn * ((a.M + kNvBM - 1) / kNvBM);
  const int my_tiles = (long long)blockIdx.x < ntiles ? (int)((ntiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;

  // The second weight-scale half of a stage is not loaded for a tile whose
  // second 128 columns lie past N (those weight rows are TMA zero fill); zero
  // it once so that it never holds a NaN pattern (later tiles leave finite scales).
  for (int i = threadIdx.x; i < kNvStages * 128; i += blockDim.x) {
    const int s = i >> 7, q = i & 127;
    reinterpret_cast<uint4*>(sm + s * kNvStageBytes + kNvABytes + kNvBBytes + kNvSfaBytes + 2048)[q] =
        make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kNvStages; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(&bar_acc_full, 1);
    mbar_init(&bar_acc_empty, kNvEpiWarps);
    mbar_init(&bar_drain, 1);
    abort_flag = 0;
    never_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, kNvTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ================= loads =================
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      bool ok = true;
      long long it = 0;  // ring position over all of this CTA's stages
      for (int i = 0; i < my_tiles && ok; ++i) {
        const long long t = blockIdx.x + (long long)i * gridDim.x;
        const int nt = (int)(t % ntn), mt = (int)(t / ntn);
        const bool has_b1 = 2 * nt + 1 < nt128;
        const uint32_t tx = kNvABytes + kNvBBytes + kNvSfaBytes + (has_b1 ? 2u : 1u) * 2048u;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = (int)(it % kNvStages);
          if (it >= kNvStages) {
            ok = mbar_wait(&bar_empty[s], (uint32_t)((it / kNvStages) - 1) & 1u, &abort_flag, a.limit_ns);
            if (!ok) break;
          }
          uint8_t* st = sm + s * kNvStageBytes;
          mbar_arrive_expect_tx(&bar_full[s], tx);
          tma_load_2d(st, &tmA, &bar_full[s], kb * 128, mt * kNvBM);
          tma_load_2d(st + kNvABytes, &tmB, &bar_full[s], kb * 128, nt * kNvBN);
          bulk_load(st + kNvABytes + kNvBBytes, a.sfa + ((long long)mt * KS + kb * 4) * 512, kNvSfaBytes,
                    &bar_full[s]);
          bulk_load(st + kNvABytes + kNvBBytes + kNvSfaBytes, a.sfb + ((long long)(2 * nt) * KS + kb * 4) * 512, 2048,
                    &bar_full[s]);
          if (has_b1)
            bulk_load(st + kNvABytes + kNvBBytes + kNvSfaBytes + 2048,
                      a.sfb + ((long long)(2 * nt + 1) * KS + kb * 4) * 512, 2048, &bar_full[s]);
        }
      }
      if (!ok) {
        abort_flag = 1;
        report_error(-6);
      }
      // drain: every issued load lands before the CTA may exit
      for (long long j = it > kNvStages ? it - kNvStages : 0; j < it; ++j)
        mbar_wait(&bar_full[j % kNvStages], (uint32_t)(j / kNvStages) & 1u, &never_abort, a.limit_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ================= scales -> TMEM, MMA =================
      bool ok = true;
      long long it = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        if (i > 0) {  // the epilogue has read the previous tile's accumulator
          ok = mbar_wait(&bar_acc_empty, (uint32_t)(i - 1) & 1u, &abort_flag, a.limit_ns);
          if (!ok) break;
          tc_fence_after();
        }
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = (int)(it % kNvStages);
          ok = mbar_wait(&bar_full[s], (uint32_t)(it / kNvStages) & 1u, &abort_flag, a.limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = smem_u32(sm + s * kNvStageBytes);
          const uint32_t sfa_s = st + kNvABytes + kNvBBytes, sfb_s = sfa_s + kNvSfaBytes;
          const uint32_t tsf = tb + 256u + (uint32_t)s * 48u;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t ta = tsf + kk * 4u, tbs = tsf + 16u + kk * 8u;
            tmem_cp_32x128b_x4(ta, smem_desc(sfa_s + kk * 512u, 128, 128, SW_NONE));
            tmem_cp_32x128b_x4(tbs, smem_desc(sfb_s + kk * 512u, 128, 128, SW_NONE));
            tmem_cp_32x128b_x4(tbs + 4u, smem_desc(sfb_s + 2048u + kk * 512u, 128, 128, SW_NONE));
            mma_nvf4(tb, smem_desc(st + kk * 32u, 16, 1024, SW_128B),
                     smem_desc(st + kNvABytes + kk * 32u, 16, 1024, SW_128B), kNvIdesc, ta, tbs,
                     (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&bar_empty[s]);
        }
        if (ok) mma_commit(&bar_acc_full);
      }
      if (!ok) {
        abort_flag = 1;
        report_error(-6);
      }
      // drain: every issued MMA completes before TMEM is released
      mma_commit(&bar_drain);
      mbar_wait(&bar_drain, 0, &never_abort, a.limit_ns);
    }
    __syncwarp();
  } else {
    // ================= epilogue: TMEM -> registers -> alpha, bias -> bf16 =================
    const int et = threadIdx.x - 64;                  // 0 .. 32*kNvEpiWarps-1
    const int q = warp & 3, half = (warp - 2) >> 2;   // TMEM lane quarter; column half
    const uint32_t taddr = tb + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 128);
    const float alpha = __fmul_rn(*a.gx, *a.gw);
    bool ok = true;
    for (int i = 0; i < my_tiles; ++i) {  // the same count in every epilogue thread: one named barrier per tile
      const long long t = blockIdx.x + (long long)i * gridDim.x;
      const int nt = (int)(t % ntn), mt = (int)(t / ntn);
      float* sb = sbias[i & 1];
      {
        const int n = nt * kNvBN + et;
        sb[et] = (a.bias && n < a.N) ? a.bias[n] : 0.f;
      }
      named_barrier_sync(1, 32 * kNvEpiWarps);
      if (ok) ok = mbar_wait_hint(&bar_acc_full, (uint32_t)i & 1u, &abort_flag, a.limit_ns, 20000u);
      ok = __all_sync(0xFFFFFFFFu, ok && !abort_flag);  // one decision per warp: tcgen05.ld is warp-wide
      const int left = (a.N - nt * kNvBN) / 32 - half * 4;  // chunks of this half inside N (N % 128 == 0)
      const int nch = ok ? (left < 0 ? 0 : (left > 4 ? 4 : left)) : 0;
      uint32_t v0[32], v1[32], v2[32], v3[32];
      if (nch > 0) {
        tc_fence_after();
        tmem_ld32(taddr, v0);
        if (nch > 1) tmem_ld32(taddr + 32u, v1);
        if (nch > 2) tmem_ld32(taddr + 64u, v2);
        if (nch > 3) tmem_ld32(taddr + 96u, v3);
        tmem_wait_ld();
        reg_fence32(v0);
        reg_fence32(v1);
        reg_fence32(v2);
        reg_fence32(v3);
      }
      // hand the accumulator back (also after a failure, so that the counts match)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_acc_empty);
      const long long row = (long long)mt * kNvBM + q * 32 + lane;
      if (nch > 0 && row < a.M) {
        __nv_bfloat16* yrow = a.y + row * a.ldy + nt * kNvBN + half * 128;
        const float* sbh = sb + half * 128;
        nv_store_chunk(v0, sbh, alpha, yrow);
        if (nch > 1) nv_store_chunk(v1, sbh + 32, alpha, yrow + 32);
        if (nch > 2) nv_store_chunk(v2, sbh + 64, alpha, yrow + 64);
        if (nch > 3) nv_store_chunk(v3, sbh + 96, alpha, yrow + 96);
      }
    }
    if (!ok && lane == 0) report_error(-6);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, kNvTmemCols);
  }
}

}  // namespace lx
