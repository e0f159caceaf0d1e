// Planner kernels: block-mean pooling of Q and K (step a1); pooled-mean
// scores on the tensor cores and per-row top-k selection (step a2).
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
// a2, scores: S[b,h,i,j] = Mq[b,h,i,:] . Mk[b,h,j,:] for all block pairs of a
// head, on the tensor cores with fp32-level accuracy.  One 128-thread CTA
// computes a 128-row x 128-key tile; 48 KB of shared memory and 128 TMEM
// columns let four CTAs share an SM.  Each 16-dimension chunk of the pooled
// means arrives by TMA (fp32, 64-byte swizzle) into one of two chunk buffers
// (the next chunk loads while the current one is used) and is split in place
// into a tf32-exact high part h = x rounded to 10 mantissa bits, plus the
// remainder l = x - h (exact in fp32) in a third buffer; three kind::tf32
// MMAs (h.h + h.l + l.h) then accumulate in TMEM, leaving only the l.l term and the tf32 truncation of l,
// about 2^-22 of each product.  The tile leaves through shared memory, one
// 128-byte row segment per warp store; rows are ldS = nB rounded up to 32
// floats apart, so that each starts on a 128-byte boundary (columns nB..ldS-1
// are never written).  Dividing by sqrt(d) changes no ranking and is left out.
constexpr int kSgM = 128, kSgN = 128, kSgK = 16;  // rows, keys, dimensions per chunk (64-byte rows)
constexpr int kSgA = kSgM * kSgK * 4;             // bytes of one A chunk (8 KB)
constexpr int kSgB = kSgN * kSgK * 4;             // bytes of one B chunk (8 KB)
constexpr int kSgRaw = kSgA + kSgB;               // one raw chunk (A then B)
constexpr int kSgSmem = 3 * kSgRaw;              // two chunk buffers (raw, then high part) + low parts
constexpr uint32_t kSgIdesc = instr_desc(IDESC_DF32, IDESC_TF32, IDESC_TF32, 0, 0, kSgM, kSgN);

__device__ __forceinline__ float tf32_high(float v) {
  return __uint_as_float((__float_as_uint(v) + 0x1000u) & 0xFFFFE000u);
}

template <int D>
__global__ void __launch_bounds__(128, 4) score_gemm_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                           const __grid_constant__ CUtensorMap tmK,
                                                           float* __restrict__ S, int nB, int ldS,
                                                           unsigned long long limit_ns) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* raw = sm;                     // 2 x [A chunk | B chunk]: TMA destinations, then high parts
  uint8_t* lo = sm + 2 * kSgRaw;         // [A | B] low parts, same swizzled layout
  __shared__ uint64_t bar_ld[2], bar_mma;
  __shared__ uint32_t tmem_slot;
  __shared__ int never_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kSgM, n0 = blockIdx.y * kSgN, bh = blockIdx.z;
  constexpr int NK = D / kSgK;
  if (threadIdx.x == 0) {
    mbar_init(&bar_ld[0], 1);
    mbar_init(&bar_ld[1], 1);
    mbar_init(&bar_mma, 1);
    never_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, kSgN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;
  // every exit from the chunk loop is CTA-uniform (__syncthreads_and), so no
  // thread is left at a barrier; loads and MMAs in flight are drained below
  int issued_ld = 0, issued_mma = 0;  // chunks whose TMA loads / MMAs thread 0 issued
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar_ld[0], kSgRaw);
    tma_load_4d(raw, &tmQ, &bar_ld[0], 0, m0, bh, 0);
    tma_load_4d(raw + kSgA, &tmK, &bar_ld[0], 0, n0, bh, 0);
    issued_ld = 1;
  }
  bool ok = true;
  for (int kc = 0; kc < NK; ++kc) {
    const int rb = kc & 1;
    uint8_t* hi = raw + rb * kSgRaw;
    // chunk kc has landed, and the previous chunk's MMAs are done with the low
    // buffer and with the other chunk buffer, which chunk kc+1 now loads into
    bool w = mbar_wait(&bar_ld[rb], (kc >> 1) & 1, &never_abort, limit_ns);
    w = w && (kc == 0 || mbar_wait(&bar_mma, (kc - 1) & 1, &never_abort, limit_ns));
    ok = __syncthreads_and(ok && w) != 0;
    if (!ok) break;
    if (threadIdx.x == 0 && kc + 1 < NK) {
      uint8_t* nxt = raw + (rb ^ 1) * kSgRaw;
      mbar_arrive_expect_tx(&bar_ld[rb ^ 1], kSgRaw);
      tma_load_4d(nxt, &tmQ, &bar_ld[rb ^ 1], (kc + 1) * kSgK, m0, bh, 0);
      tma_load_4d(nxt + kSgA, &tmK, &bar_ld[rb ^ 1], (kc + 1) * kSgK, n0, bh, 0);
      issued_ld = kc + 2;
    }
    float4* h4 = reinterpret_cast<float4*>(hi);
    float4* l4 = reinterpret_cast<float4*>(lo);
    for (int i = threadIdx.x; i < kSgRaw / 16; i += blockDim.x) {
      const float4 x = h4[i];
      const float4 h = make_float4(tf32_high(x.x), tf32_high(x.y), tf32_high(x.z), tf32_high(x.w));
      h4[i] = h;
      l4[i] = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < kSgK / 8; ++ks) {  // 8 tf32 values = 32 bytes per MMA
        const uint64_t ah = smem_desc(smem_u32(hi) + ks * 32, 16, 8 * 64, SW_64B);
        const uint64_t al = smem_desc(smem_u32(lo) + ks * 32, 16, 8 * 64, SW_64B);
        const uint64_t bhd = smem_desc(smem_u32(hi + kSgA) + ks * 32, 16, 8 * 64, SW_64B);
        const uint64_t bld = smem_desc(smem_u32(lo + kSgA) + ks * 32, 16, 8 * 64, SW_64B);
        mma_ss<KIND_TF32>(tbase, ah, bhd, kSgIdesc, (kc > 0 || ks > 0) ? 1u : 0u);
        mma_ss<KIND_TF32>(tbase, ah, bld, kSgIdesc, 1u);
        mma_ss<KIND_TF32>(tbase, al, bhd, kSgIdesc, 1u);
      }
      mma_commit(&bar_mma);
      issued_mma = kc + 1;
    }
  }
  if (ok) ok = __syncthreads_and(mbar_wait(&bar_mma, (NK - 1) & 1, &never_abort, limit_ns)) != 0;
  if (!ok) {
    if (threadIdx.x == 0) {
      report_error(-6);
      // drain what is still in flight before the CTA exits and frees TMEM
      for (int c = issued_ld - 2 < 0 ? 0 : issued_ld - 2; c < issued_ld; ++c)
        mbar_wait(&bar_ld[c & 1], (c >> 1) & 1, &never_abort, limit_ns);
      if (issued_mma > 0) mbar_wait(&bar_mma, (issued_mma - 1) & 1, &never_abort, limit_ns);
    }
  } else {
    tc_fence_after();
    // warp w holds tile rows 32w .. 32w+31 (TMEM lanes of its quarter); each
    // 32 x 32 block goes through a padded shared tile (in the two chunk
    // buffers, idle once the last MMA is done) and out row by row, one 128-byte
    // segment per store
    static_assert(4 * 32 * 33 * 4 <= 2 * kSgRaw, "epilogue tiles exceed the chunk buffers");
    float* tile = reinterpret_cast<float*>(raw) + warp * 32 * 33;
#pragma unroll 1
    for (int cc = 0; cc < kSgN; cc += 32) {
      uint32_t v[32];
      tmem_ld32(tbase + ((uint32_t)(warp * 32) << 16) + cc, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) tile[lane * 33 + i] = __uint_as_float(v[i]);
      __syncwarp();
      const int j = n0 + cc + lane;
#pragma unroll 4
      for (int r = 0; r < 32; ++r) {
        const int row = m0 + warp * 32 + r;
        if (row < nB && j < nB) S[((long long)bh * nB + row) * ldS + j] = tile[r * 33 + lane];
      }
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kSgN);
  }
}

// ---------------------------------------------------------------------------
// a2, selection: one 256-thread CTA per (b*h, 8 query-block rows); the 8
// score rows (contiguous in the workspace, ldS floats apart) arrive in shared
// memory by one bulk copy, and each warp selects one row: scores are bucketed
// into 128 monotone buckets between the row min and max; the bucket holding
// the k-th largest is resolved exactly by ranking its members with the (score
// desc, index asc) order; the kept ids are emitted in ascending order with
// ballots that are also the bitmask words.
constexpr int kScoreRows = 8;
constexpr int kCandCap = 64;
constexpr int kScoreWarps = 8;
constexpr int kBuckets = 128;
constexpr int kMaxChunks = 17;  // 128-score chunks of the longest row (nB <= 2176)

// Bucket of a score: (s - mn) * scale clamped to [0, 127] and rounded to the
// nearest integer by adding 1.5 * 2^23 (whose float spacing is 1), then read
// from the bits.  Non-decreasing in s.  For a finite row s - mn >= 0; a NaN
// (from a NaN or infinite score) clamps to 127, so the id is always in range.
__device__ __forceinline__ uint32_t score_bucket(float s, float mn, float scale) {
  const float t = fminf((s - mn) * scale, 127.0f);
  return (__float_as_uint(t + 12582912.0f) - 0x4B400000u) & 127u;
}

// Four bucket ids packed one per byte (bit 7 of each byte clear): bit 7 of
// byte e of the result is set where id_e > y (y + 1 <= 128, so no byte borrows
// from its neighbour), or where id_e >= y for ge.
__device__ __forceinline__ uint32_t bytes_gt(uint32_t pk, uint32_t y) {
  return ((pk | 0x80808080u) - (y + 1u) * 0x01010101u) & 0x80808080u;
}
__device__ __forceinline__ uint32_t bytes_ge(uint32_t pk, uint32_t y) {
  return ((pk | 0x80808080u) - y * 0x01010101u) & 0x80808080u;
}
// Bit 7 of byte e -> bit e (the four products land on bits 28..31 and
// nowhere else below 32).
__device__ __forceinline__ uint32_t high_bits_to_nibble(uint32_t m) { return ((m >> 7) * 0x10204080u) >> 28; }

// Select the k best keys of one score row (warp-wide) and write the ascending
// ids (and the bitmask words when `mask` is not null).  Returns the number of
// ids selected (k unless the row holds non-finite scores).  The row is walked
// in chunks of 128 scores; lane l holds scores j = 128c + 32e + l (e = 0..3),
// so that one ballot per e is one 32-bit mask word.  The histogram pass keeps
// the four bucket ids of each lane and chunk in a register (pk[c]); the chunk
// loops are unrolled to kMaxChunks so that pk stays in registers.  The ids are
// gathered in the row's own shared buffer (no longer read once the ranking is
// done) and the mask words in `selbits`, and both leave in coalesced stores.
__device__ int select_row(float* s, int nB, int k, int* hist, float* cand_s, int* cand_j, uint32_t* selbits,
                          int32_t* __restrict__ idx_out, uint32_t* __restrict__ mask_out) {
  const int lane = threadIdx.x & 31;
  const int nC = (nB + 127) >> 7;
  __syncwarp();
  float mn = INFINITY, mx = -INFINITY;
  for (int ch = 0; ch < nC; ++ch) {
    const int j0 = 128 * ch + 4 * lane;
    if (j0 + 4 <= nB) {
      const float4 v = *reinterpret_cast<const float4*>(s + j0);
      mn = fminf(mn, fminf(fminf(v.x, v.y), fminf(v.z, v.w)));
      mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    } else {
      for (int j = j0; j < nB; ++j) {
        mn = fminf(mn, s[j]);
        mx = fmaxf(mx, s[j]);
      }
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  const int nW = (nB + 31) >> 5;
  for (int w = lane; w < nW; w += 32) selbits[w] = 0u;
  uint32_t bt = 0;
  int need = k;
  uint32_t pk[kMaxChunks];
#pragma unroll
  for (int ch = 0; ch < kMaxChunks; ++ch) pk[ch] = 0u;
  const bool flat = !(mx > mn);  // all equal (or non-finite): lowest ids win
  if (!flat) {
    const float scale = 127.99f / (mx - mn);
    for (int i = lane; i < kBuckets; i += 32) hist[i] = 0;
    __syncwarp();
#pragma unroll
    for (int ch = 0; ch < kMaxChunks; ++ch) {
      if (ch >= nC) break;
      const int rem = nB - 128 * ch - lane;  // score e of this lane exists while 32e < rem
      uint32_t p = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (32 * e < rem) {
          const uint32_t b = score_bucket(s[128 * ch + 32 * e + lane], mn, scale);
          atomicAdd(&hist[b], 1);
          p |= b << (8 * e);
        }
      }
      pk[ch] = p;
    }
    __syncwarp();
    // lane l owns buckets 127-4l .. 124-4l (descending); find the bucket holding rank k
    int cnt[4], tot = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      cnt[i] = hist[kBuckets - 1 - 4 * lane - i];
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
      for (int i = 0; i < 4; ++i) {
        if (my_bt < 0) {
          if (above + cnt[i] >= k) {
            my_bt = kBuckets - 1 - 4 * lane - i;
            my_need = k - above;
          } else {
            above += cnt[i];
          }
        }
      }
    }
    bt = (uint32_t)__shfl_sync(0xffffffffu, my_bt, owner);
    need = __shfl_sync(0xffffffffu, my_need, owner);
    // members of bucket bt, ranked by (score desc, index asc)
    const int c = hist[bt];
    if (c <= kCandCap) {
      // membership words: word 4c + e is the ballot of score e of chunk c
      // (ids 32 (4c + e) + lane); lane l keeps words l, l + 32 and l + 64
      uint32_t wk[3] = {0u, 0u, 0u};
#pragma unroll
      for (int ch = 0; ch < kMaxChunks; ++ch) {
        if (ch >= nC) break;
        const int rem = nB - 128 * ch - lane;
        const uint32_t valid = (1u << (rem <= 0 ? 0 : min(4, (rem + 31) >> 5))) - 1u;
        const uint32_t m = high_bits_to_nibble(bytes_ge(pk[ch], bt) & ~bytes_gt(pk[ch], bt)) & valid;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t b = __ballot_sync(0xffffffffu, (m >> e) & 1u);
          if (lane == ((4 * ch + e) & 31)) wk[(4 * ch + e) >> 5] = b;
        }
      }
      // each lane expands its words, ascending, at the offset given by the
      // popcounts of the words before it
      int base = 0;
#pragma unroll
      for (int g = 0; g < 3; ++g) {
        if (32 * g >= nW) break;
        uint32_t mm = wk[g];
        const int cnt = __popc(mm);
        int incl = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += v;
        }
        int pos = base + incl - cnt;
        while (mm) {
          const int j = 32 * (32 * g + lane) + __ffs(mm) - 1;
          mm &= mm - 1;
          cand_s[pos] = s[j];
          cand_j[pos] = j;
          ++pos;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
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
  // the mask words first: word 4c + e is the ballot of score e of the lanes in
  // chunk c, and replaces selbits word 4c + e once every lane has read it
#pragma unroll
  for (int ch = 0; ch < kMaxChunks; ++ch) {
    if (ch >= nC) break;
    const int rem = nB - 128 * ch - lane;
    const int ne = rem <= 0 ? 0 : min(4, (rem + 31) >> 5);  // scores of this lane in the chunk
    const uint32_t valid = (1u << ne) - 1u;
    uint32_t sel;
    if (flat) {
      const int remk = min(k, nB) - 128 * ch - lane;
      sel = (1u << (remk <= 0 ? 0 : min(4, (remk + 31) >> 5))) - 1u;
    } else {
      const uint32_t gt = bytes_gt(pk[ch], bt);
      sel = high_bits_to_nibble(gt) & valid;
      uint32_t eq = high_bits_to_nibble(bytes_ge(pk[ch], bt) & ~gt) & valid;
      while (eq) {
        const int e = __ffs(eq) - 1;
        eq &= eq - 1;
        sel |= ((selbits[4 * ch + e] >> lane) & 1u) << e;
      }
    }
    const uint32_t b0 = __ballot_sync(0xffffffffu, sel & 1u), b1 = __ballot_sync(0xffffffffu, sel & 2u);
    const uint32_t b2 = __ballot_sync(0xffffffffu, sel & 4u), b3 = __ballot_sync(0xffffffffu, sel & 8u);
    if (lane < 4 && 4 * ch + lane < nW) selbits[4 * ch + lane] = lane == 0 ? b0 : (lane == 1 ? b1 : (lane == 2 ? b2 : b3));
  }
  __syncwarp();
  // then the ids, ascending, into the row buffer (no longer read): lane l
  // expands word w0 + l at the offset given by the popcounts of the words before it
  int* ids = reinterpret_cast<int*>(s);
  int written = 0;
  for (int w0 = 0; w0 < nW; w0 += 32) {
    const int w = w0 + lane;
    uint32_t m = w < nW ? selbits[w] : 0u;
    const int cnt = __popc(m);
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int pos = written + incl - cnt;
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1;
      if (pos < k) ids[pos] = 32 * w + b;
      ++pos;
    }
    written += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncwarp();
  const int n_out = min(written, k);
  for (int i = lane; i < n_out; i += 32) idx_out[i] = ids[i];
  if (mask_out)
    for (int w = lane; w < nW; w += 32) mask_out[w] = selbits[w];
  return written;
}

__global__ void __launch_bounds__(32 * kScoreWarps) select_topk_kernel(const float* __restrict__ S, int nB, int k,
                                                                      int32_t* __restrict__ idx,
                                                                      uint32_t* __restrict__ mask, int ldS,
                                                                      unsigned long long limit_ns) {
  extern __shared__ __align__(16) float smem_f[];
  float* sS = smem_f;                                                        // [8][ldS]
  int* hist = reinterpret_cast<int*>(sS + kScoreRows * ldS);                 // warps x 128
  float* cand_s = reinterpret_cast<float*>(hist + kScoreWarps * kBuckets);  // warps x 64
  int* cand_j = reinterpret_cast<int*>(cand_s + kScoreWarps * kCandCap);    // warps x 64
  uint32_t* selbits = reinterpret_cast<uint32_t*>(cand_j + kScoreWarps * kCandCap);  // warps x ldS/32
  __shared__ uint64_t bar_ld;
  __shared__ int never_abort;
  const long long bh = blockIdx.y;
  const int row0 = blockIdx.x * kScoreRows;
  const int nrows = min(kScoreRows, nB - row0);
  // nrows * ldS * 4 bytes: a multiple of 128, from a 128-byte aligned row
  const uint32_t bytes = (uint32_t)(nrows * ldS) * 4u;
  if (threadIdx.x == 0) {
    mbar_init(&bar_ld, 1);
    never_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar_ld, bytes);
    bulk_load(sS, S + (bh * nB + row0) * (long long)ldS, bytes, &bar_ld);
  }
  // one thread waits (suspending between polls, so that the waiting CTA takes
  // no issue slots from the CTAs that compute); after the barrier every thread
  // observes the completed phase itself, which makes the copied rows visible to it
  bool landed = true;
  if (threadIdx.x == 0) landed = mbar_wait_hint(&bar_ld, 0, &never_abort, limit_ns, 20000u);
  if (__syncthreads_and(landed) == 0) {
    // the copy did not land in time: wait (bounded) for it before the CTA exits
    if (threadIdx.x == 0) {
      report_error(-6);
      mbar_wait(&bar_ld, 0, &never_abort, limit_ns);
    }
    return;
  }
  if (!mbar_try_wait(&bar_ld, 0)) report_error(-6);  // cannot fail: the phase has completed
  const int warp = threadIdx.x >> 5;
  const int nW = (nB + 31) >> 5;
  for (int r = warp; r < nrows; r += kScoreWarps) {
    const long long row = bh * nB + row0 + r;
    const int got = select_row(sS + r * ldS, nB, k, hist + warp * kBuckets, cand_s + warp * kCandCap,
                               cand_j + warp * kCandCap, selbits + warp * (ldS / 32),
                               idx + row * k, mask ? mask + row * nW : nullptr);
    if (got != k && (threadIdx.x & 31) == 0) {
      report_error(-7);  // non-finite scores: the row could not be ordered
      for (int p = got; p < k; ++p) idx[row * k + p] = -1;
    }
  }
}

}  // namespace lx
