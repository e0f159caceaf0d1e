// Planner kernels: block-mean pooling of Q and K (step a1) and pooled-mean
// scoring with per-row top-k selection (step a2).
//
// "600倍加速，720p视频实时生成！单卡也能带的动14B模型", §动态稀疏量化注意力: the
// importance of each attention tile is estimated from block-level means of Q
// and K and the key blocks are chosen at run time.  The 64-token block, the
// score s[i,j] = mean(Q_i).mean(K_j)/sqrt(d) and the top-ceil(keep*nB) rule
// with ties to the lower index are this library's reading of that sentence.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "ptx.cuh"

namespace lx {

constexpr int kBlock = 64;

struct BhldView {  // bf16 [B,H,L,D] with element strides (stride of D is 1)
  const __nv_bfloat16* p;
  long long sB, sH, sL;
};

__device__ __forceinline__ uint4 ld_stream_v4(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] += __uint_as_float(w[i] << 16);
    a[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// ---------------------------------------------------------------------------
// a1: one warp per (tensor, b*h, block).  Lanes split a row into 16-byte chunks
// (D/8 lanes per row); the warp walks the block's valid rows with 128-bit
// streaming loads, accumulates in fp32, folds the lanes that share a chunk and
// divides by the number of valid tokens.  Output fp32 [B*H, nB, D].
template <int D>
__global__ void __launch_bounds__(256) pool_means_kernel(BhldView q, BhldView k, float* __restrict__ mq,
                                                        float* __restrict__ mk, int H, int L, int nB,
                                                        long long units) {
  constexpr int CH = D / 8;          // 16-byte chunks per row
  constexpr int RPI = 32 / CH;       // rows per warp iteration
  constexpr int ITERS = kBlock / RPI;
  constexpr int UNROLL = 8;
  const long long unit = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (unit >= units) return;
  const int lane = threadIdx.x & 31;
  const BhldView X = blockIdx.y == 0 ? q : k;
  float* __restrict__ M = blockIdx.y == 0 ? mq : mk;
  const long long bh = unit / nB;
  const int blk = (int)(unit - bh * nB);
  const long long b = bh / H, h = bh - b * H;
  const int t0 = blk * kBlock;
  const int cnt = min(kBlock, L - t0);
  const int c = lane % CH, ro = lane / CH;
  const __nv_bfloat16* base = X.p + b * X.sB + h * X.sH + (long long)t0 * X.sL + c * 8;
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
  for (int it0 = 0; it0 < ITERS; it0 += UNROLL) {
    uint4 v[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int row = (it0 + u) * RPI + ro;
      v[u] = row < cnt ? ld_stream_v4(base + (long long)row * X.sL) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) acc_bf16x8(a, v[u]);
  }
#pragma unroll
  for (int off = CH; off < 32; off <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] += __shfl_xor_sync(0xffffffffu, a[i], off);
  if (ro == 0) {
    const float n = (float)cnt;
    float4* out = reinterpret_cast<float4*>(M + (bh * nB + blk) * D + c * 8);
    out[0] = make_float4(__fdiv_rn(a[0], n), __fdiv_rn(a[1], n), __fdiv_rn(a[2], n), __fdiv_rn(a[3], n));
    out[1] = make_float4(__fdiv_rn(a[4], n), __fdiv_rn(a[5], n), __fdiv_rn(a[6], n), __fdiv_rn(a[7], n));
  }
}

// ---------------------------------------------------------------------------
// a2: one CTA per (b*h, 16 query-block rows), 16 warps.
//  Scoring: every warp computes all 16 rows for its share of the key blocks
//  (two keys at a time, so eight independent FMA chains per lane).
//  Lane = (row group rg in 0..3) x (d-slice ds in 0..7); a lane keeps the 4
//  rows x D/8 pooled-query values of its slice in registers and reads the
//  pooled key in 16-byte pieces (slices are interleaved so the 8 slices of one
//  key are one contiguous 128-byte wavefront); partial dots are folded across
//  the 8 slices with 4 shuffles.  Scores land in shared memory (fp32).
//  Selection: one warp per row.  Scores are bucketed into 256 monotone
//  buckets between the row min and max; the bucket holding the k-th largest is
//  resolved exactly by ranking its members with the (score desc, index asc)
//  order; the kept ids are emitted in ascending order with a ballot scan that
//  also yields the bitmask words.
constexpr int kScoreRows = 16;
constexpr int kKeyChunk = 32;
constexpr int kCandCap = 64;

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Pooled keys stream through a ring of shared-memory stages filled by bulk
// copies (one thread issues, every warp reads), so the L2 latency of one chunk
// hides behind the arithmetic on the previous ones.
constexpr int kKeyStages = 3;
constexpr int kScoreWarps = 16;  // 512 threads share one CTA's score rows

template <int D>
__device__ __forceinline__ void score_rows(const float* __restrict__ Mq, const float* __restrict__ Mk, int nB,
                                           int row0, int nrows, float* sS, int ldS, float* sK, uint64_t* kfull,
                                           uint64_t* kempty, const volatile int* abort_flag,
                                           unsigned long long limit_ns) {
  constexpr int DS = D / 8;   // values per lane slice
  constexpr int NQ = DS / 4;  // float4 pieces per slice
  constexpr int CHUNK_FLOATS = kKeyChunk * D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = lane >> 3, ds = lane & 7;
  const int nchunks = (nB + kKeyChunk - 1) / kKeyChunk;
  // Slice ds covers d = 32*qq + 4*ds + e  (qq < NQ, e < 4).
  float qv[4][DS];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = row0 + rg * 4 + r;
#pragma unroll
    for (int qq = 0; qq < NQ; ++qq) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (row - row0 < nrows) v = *reinterpret_cast<const float4*>(Mq + (long long)row * D + 32 * qq + 4 * ds);
      qv[r][4 * qq] = v.x;
      qv[r][4 * qq + 1] = v.y;
      qv[r][4 * qq + 2] = v.z;
      qv[r][4 * qq + 3] = v.w;
    }
  }
  auto issue = [&](int ch) {
    const int st = ch % kKeyStages;
    const int nk = min(kKeyChunk, nB - ch * kKeyChunk);
    mbar_arrive_expect_tx(&kfull[st], (uint32_t)(nk * D * 4));
    bulk_load(sK + st * CHUNK_FLOATS, Mk + (long long)ch * kKeyChunk * D, (uint32_t)(nk * D * 4), &kfull[st]);
  };
  if (threadIdx.x == 0)
    for (int ch = 0; ch < min(kKeyStages, nchunks); ++ch) issue(ch);
  bool ok = true;
  for (int ch = 0; ch < nchunks; ++ch) {
    const int st = ch % kKeyStages;
    const int j0 = ch * kKeyChunk;
    const int nk = min(kKeyChunk, nB - j0);
    if (!mbar_wait(&kfull[st], (ch / kKeyStages) & 1, abort_flag, limit_ns)) {
      ok = false;
      break;
    }
    const float* sKc = sK + st * CHUNK_FLOATS;
    // warp w handles keys jj = w and w + 16 of the chunk, together
    {
      const int ja = warp, jb = warp + kScoreWarps;
      const bool va = ja < nk, vb = jb < nk;
      const float* ka = sKc + (va ? ja : 0) * D;
      const float* kb = sKc + (vb ? jb : 0) * D;
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int qq = 0; qq < NQ; ++qq) {
        const float4 xa = *reinterpret_cast<const float4*>(ka + 32 * qq + 4 * ds);
        const float4 xb = *reinterpret_cast<const float4*>(kb + 32 * qq + 4 * ds);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          acc[0][r] = fmaf(qv[r][4 * qq], xa.x, acc[0][r]);
          acc[1][r] = fmaf(qv[r][4 * qq], xb.x, acc[1][r]);
          acc[0][r] = fmaf(qv[r][4 * qq + 1], xa.y, acc[0][r]);
          acc[1][r] = fmaf(qv[r][4 * qq + 1], xb.y, acc[1][r]);
          acc[0][r] = fmaf(qv[r][4 * qq + 2], xa.z, acc[0][r]);
          acc[1][r] = fmaf(qv[r][4 * qq + 2], xb.z, acc[1][r]);
          acc[0][r] = fmaf(qv[r][4 * qq + 3], xa.w, acc[0][r]);
          acc[1][r] = fmaf(qv[r][4 * qq + 3], xb.w, acc[1][r]);
        }
      }
      // fold the 8 slices: after three stages lane ds holds row 2*(ds>>2&1)+(ds>>1&1)
      const bool hi4 = (ds & 4) != 0, hi2 = (ds & 2) != 0;
      const int r = 2 * (hi4 ? 1 : 0) + (hi2 ? 1 : 0);
#pragma unroll
      for (int kx = 0; kx < 2; ++kx) {
        float s0 = hi4 ? acc[kx][0] : acc[kx][2], s1 = hi4 ? acc[kx][1] : acc[kx][3];
        float k0 = hi4 ? acc[kx][2] : acc[kx][0], k1 = hi4 ? acc[kx][3] : acc[kx][1];
        k0 += __shfl_xor_sync(0xffffffffu, s0, 4);
        k1 += __shfl_xor_sync(0xffffffffu, s1, 4);
        float s2 = hi2 ? k0 : k1;
        float k2 = hi2 ? k1 : k0;
        k2 += __shfl_xor_sync(0xffffffffu, s2, 2);
        k2 += __shfl_xor_sync(0xffffffffu, k2, 1);
        const int jj = kx ? jb : ja;
        if ((ds & 1) == 0 && (kx ? vb : va)) sS[(rg * 4 + r) * ldS + j0 + jj] = k2;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&kempty[st]);
    // refill this stage with chunk ch + kKeyStages once all warps are done with it
    if (threadIdx.x == 0 && ch + kKeyStages < nchunks) {
      if (!mbar_wait(&kempty[st], (ch / kKeyStages) & 1, abort_flag, limit_ns)) {
        ok = false;
        break;
      }
      issue(ch + kKeyStages);
    }
  }
  if (!ok) report_error(-6);
  __syncthreads();
}

__device__ __forceinline__ int score_bucket(float s, float mn, float scale) {
  float t = (s - mn) * scale;
  int b = (int)t;  // t >= 0 for finite s >= mn; NaN converts to 0
  return min(255, max(0, b));
}

// Select the k best keys of one score row (warp-wide) and write the ascending
// ids (and the bitmask words when `mask` is not null).  Returns the number of
// ids written (k unless the row holds non-finite scores).
__device__ int select_row(const float* __restrict__ s, int nB, int k, int* hist, float* cand_s, int* cand_j,
                          uint32_t* selbits, int32_t* __restrict__ idx_out, uint32_t* __restrict__ mask_out) {
  const int lane = threadIdx.x & 31;
  float mn = INFINITY, mx = -INFINITY;
  for (int j = lane; j < nB; j += 32) {
    mn = fminf(mn, s[j]);
    mx = fmaxf(mx, s[j]);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  const int nW = (nB + 31) >> 5;
  for (int w = lane; w < nW; w += 32) selbits[w] = 0u;
  int bt = 0, need = k;
  float scale = 0.f;
  const bool flat = !(mx > mn);  // all equal (or non-finite): lowest ids win
  if (!flat) {
    scale = 255.99f / (mx - mn);
    for (int i = lane; i < 256; i += 32) hist[i] = 0;
    __syncwarp();
    for (int j = lane; j < nB; j += 32) atomicAdd(&hist[score_bucket(s[j], mn, scale)], 1);
    __syncwarp();
    // lane l owns buckets 255-8l .. 248-8l (descending); find the bucket holding rank k
    int cnt[8], tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      cnt[i] = hist[255 - 8 * lane - i];
      tot += cnt[i];
    }
    int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    const int excl = incl - tot;
    // k <= nB keys are all counted, so exactly one lane holds the crossing
    const uint32_t hit = __ballot_sync(0xffffffffu, excl < k && incl >= k);
    const int owner = __ffs(hit) - 1;
    int my_bt = -1, my_need = 0;
    if (lane == owner) {
      int above = excl;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (my_bt < 0) {
          if (above + cnt[i] >= k) {
            my_bt = 255 - 8 * lane - i;
            my_need = k - above;
          } else {
            above += cnt[i];
          }
        }
      }
    }
    bt = __shfl_sync(0xffffffffu, my_bt, owner);
    need = __shfl_sync(0xffffffffu, my_need, owner);
    // members of bucket bt, ranked by (score desc, index asc)
    const int c = hist[bt];
    if (c <= kCandCap) {
      int base = 0;
      for (int j0 = 0; j0 < nB; j0 += 32) {
        const int j = j0 + lane;
        const bool in = j < nB && score_bucket(s[j], mn, scale) == bt;
        const uint32_t bal = __ballot_sync(0xffffffffu, in);
        if (in) {
          const int pos = base + __popc(bal & lanemask_lt());
          cand_s[pos] = s[j];
          cand_j[pos] = j;
        }
        base += __popc(bal);
      }
      __syncwarp();
      for (int i = lane; i < c; i += 32) {
        const float si = cand_s[i];
        const int ji = cand_j[i];
        int rank = 0;
        for (int t = 0; t < c; ++t) {
          const float st = cand_s[t];
          rank += (st > si) || (st == si && cand_j[t] < ji);
        }
        if (rank < need) atomicOr(&selbits[ji >> 5], 1u << (ji & 31));
      }
    } else {
      // large tie group: rank every member against the whole row (slow, exact)
      for (int j0 = 0; j0 < nB; j0 += 32) {
        const int j = j0 + lane;
        const bool in = j < nB && score_bucket(s[j], mn, scale) == bt;
        uint32_t bal = __ballot_sync(0xffffffffu, in);
        while (bal) {
          const int src = __ffs(bal) - 1;
          bal &= bal - 1;
          const int jc = j0 + src;
          const float sc = s[jc];
          int rank = 0;
          for (int t = lane; t < nB; t += 32) {
            const float st = s[t];
            rank += (score_bucket(st, mn, scale) == bt) && ((st > sc) || (st == sc && t < jc));
          }
          rank = __reduce_add_sync(0xffffffffu, rank);
          if (lane == 0 && rank < need) selbits[jc >> 5] |= 1u << (jc & 31);
        }
      }
    }
    __syncwarp();
  }
  // emit ascending ids
  int written = 0;
  for (int j0 = 0; j0 < nB; j0 += 32) {
    const int j = j0 + lane;
    bool sel = false;
    if (j < nB) {
      if (flat)
        sel = j < k;
      else {
        const int bk = score_bucket(s[j], mn, scale);
        sel = bk > bt || (bk == bt && ((selbits[j >> 5] >> (j & 31)) & 1u));
      }
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, sel);
    const int pos = written + __popc(bal & lanemask_lt());
    if (sel && pos < k) idx_out[pos] = j;
    if (mask_out && lane == 0) mask_out[j0 >> 5] = bal;
    written += __popc(bal);
  }
  return written;
}

template <int D>
__global__ void __launch_bounds__(512, 1) score_topk_kernel(const float* __restrict__ Mq, const float* __restrict__ Mk,
                                                           int nB, int k, int32_t* __restrict__ idx,
                                                           uint32_t* __restrict__ mask, int ldS,
                                                           unsigned long long limit_ns) {
  extern __shared__ __align__(16) float smem_f[];
  float* sK = smem_f;                                              // kKeyStages x [32][D]
  float* sS = sK + kKeyStages * kKeyChunk * D;                     // [16][ldS]
  int* hist = reinterpret_cast<int*>(sS + kScoreRows * ldS);                 // warps x 256
  float* cand_s = reinterpret_cast<float*>(hist + kScoreWarps * 256);       // warps x 64
  int* cand_j = reinterpret_cast<int*>(cand_s + kScoreWarps * kCandCap);    // warps x 64
  uint32_t* selbits = reinterpret_cast<uint32_t*>(cand_j + kScoreWarps * kCandCap);  // warps x ldS/32
  __shared__ uint64_t kfull[kKeyStages], kempty[kKeyStages];
  __shared__ int never_abort;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kKeyStages; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], kScoreWarps);
    }
    never_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const long long bh = blockIdx.y;
  const int row0 = blockIdx.x * kScoreRows;
  const int nrows = min(kScoreRows, nB - row0);
  score_rows<D>(Mq + bh * nB * D, Mk + bh * nB * D, nB, row0, nrows, sS, ldS, sK, kfull, kempty, &never_abort,
                limit_ns);
  const int warp = threadIdx.x >> 5;
  const int nW = (nB + 31) >> 5;
  for (int r = warp; r < nrows; r += kScoreWarps) {
    const long long row = bh * nB + row0 + r;
    const int got = select_row(sS + r * ldS, nB, k, hist + warp * 256, cand_s + warp * kCandCap,
                               cand_j + warp * kCandCap, selbits + warp * (ldS / 32), idx + row * k,
                               mask ? mask + row * nW : nullptr);
    if (got != k && (threadIdx.x & 31) == 0) {
      report_error(-7);  // non-finite scores: the row could not be ordered
      for (int p = got; p < k; ++p) idx[row * k + p] = -1;
    }
  }
}

}  // namespace lx
