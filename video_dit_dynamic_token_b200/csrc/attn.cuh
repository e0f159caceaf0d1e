// Sparse attention over the kept key blocks (step a4), tcgen05 + TMA + TMEM.
//
// "600倍加速，720p视频实时生成！单卡也能带的动14B模型", §动态稀疏量化注意力: only the
// activated attention tiles are computed and a chosen block stays dense
// inside; §高效推理算子: Q/K INT8 and V FP8.  "Run Wan2.2-A14B on One RTX 5090:
// 720p Video in 3.8s", §3 Dynamic sparse attention: the same in English.
//
// Tile: one CTA owns two adjacent 64-row query blocks (2p, 2p+1) = 128 rows,
// the full-rate M of a single-CTA tcgen05 MMA, and walks the ascending UNION of
// their two kept lists one 64-key block at a time.  A row whose own list does
// not hold the current block gets P = 0 for it and leaves its running max and
// sum untouched, so every row sees exactly its kept blocks in ascending order.
//
// Roles (6 warps): warp 0 = TMA producer (Q once, then K/V of each union block
// into a ring of stages); warp 1 = TMEM allocator + MMA issuer
// (S = Q K^T into one of two TMEM S buffers, then O += P V into the TMEM O
// accumulator); warps 2..5 = softmax / correction / epilogue, one thread per
// query row (a warp reads the TMEM lane quarter warp%4).
//
// INT8/FP8 mode follows the P-quantisation protocol: per 64-key block c the
// row max becomes m_c = max(m_{c-1}, max S_c); P~ = E4M3(448 exp(S_c - m_c));
// the accumulator and the fp32 sum of the unquantised 448*exp(S_c - m_c) are
// rescaled by exp(m_{c-1} - m_c); O = acc * sv[channel] / sum.
// BF16 mode: P = bf16(exp(S - m)), O = acc / sum.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "planner.cuh"
#include "quant.cuh"

namespace lx {

template <int D, bool I8>
struct AttnCfg {
  static constexpr int ESZ = I8 ? 1 : 2;                 // bytes per Q/K/V element
  static constexpr int ROWB = D * ESZ;                    // bytes per token row
  static constexpr int ATOM = ROWB >= 128 ? 128 : ROWB;   // swizzle atom width (128 or 64 bytes)
  static constexpr int NATOM = ROWB / ATOM;               // atom columns per row
  static constexpr int Q_BYTES = 128 * ROWB;
  static constexpr int KV_BYTES = 64 * ROWB;              // one K (or V) block
  static constexpr int NSTAGE = I8 ? 5 : 3;   // INT8: two CTAs fit one SM
  static constexpr uint32_t SW_QKV = ATOM == 128 ? SW_128B : SW_64B;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NSTAGE * KV_BYTES;
  static constexpr int OFF_MASK = OFF_V + NSTAGE * KV_BYTES;  // two bitmask rows, then (INT8) the K block scales
  static constexpr int P_COLS = 64 * ESZ / 4;             // P of one 64-key block: 16 (E4M3) or 32 (bf16) cols
  static constexpr int S_COL = 0;                         // TMEM: S tile, cols [0, 64)
  static constexpr int P_COL = 64;                        // TMEM: two P buffers, P_COLS each
  static constexpr int O_COL = 128;                       // TMEM: O accumulator, D cols
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t IDESC_S =
      instr_desc(I8 ? IDESC_DS32 : IDESC_DF32, I8 ? IDESC_S8 : IDESC_BF16, I8 ? IDESC_S8 : IDESC_BF16, 0, 0, 128, 64);
  static constexpr uint32_t IDESC_PV =
      instr_desc(IDESC_DF32, I8 ? IDESC_E4M3 : IDESC_BF16, I8 ? IDESC_E4M3 : IDESC_BF16, 0, 1, 128, D);
  static constexpr int KEYS_PER_MMA = 32 / ESZ;           // 32 bytes of K per instruction
};

struct AttnParams {
  const int32_t* idx;     // [B*H, nB, k] ascending kept ids
  int k, nB, L, H;
  __nv_bfloat16* o;       // output, element strides below (stride of D is 1)
  long long osB, osH, osL;
  const float* sq;        // INT8/FP8 mode: [B*H, nB] Q block scales
  const float* sk;        // [B*H, nB] K block scales
  const float* sv;        // [B*H, D] V channel scales
  float scale_log2;       // log2(e)/sqrt(d)
  unsigned long long limit_ns;  // bound on every wait
};

struct UnionWalk {
  const uint32_t* m0;
  const uint32_t* m1;
  int nW, w;
  uint32_t rem;
  __device__ __forceinline__ void init(const uint32_t* a, const uint32_t* b, int n) {
    m0 = a;
    m1 = b;
    nW = n;
    w = 0;
    rem = n > 0 ? (a[0] | b[0]) : 0u;
  }
  __device__ __forceinline__ bool next(int& j, int& flags) {
    while (rem == 0u) {
      if (++w >= nW) return false;
      rem = m0[w] | m1[w];
    }
    const int bit = __ffs(rem) - 1;
    rem &= rem - 1u;
    j = w * 32 + bit;
    flags = (int)((m0[w] >> bit) & 1u) | ((int)((m1[w] >> bit) & 1u) << 1);
    return true;
  }
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 12582912 = 1.5 * 2^23: an int32 s with |s| < 2^22 added to this float's bit
// pattern gives the float 12582912 + s exactly.  The INT8 score accumulator is
// started at this pattern, so the s32 QK^T result reads directly as a float.
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr float kMagic = 12582912.0f;
constexpr float kLog2_448 = 8.807354922057604f;

template <int D, bool I8>
__global__ void __launch_bounds__(192, I8 ? 2 : 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams prm) {
  using C = AttnCfg<D, I8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_q, bar_full[C::NSTAGE], bar_empty[C::NSTAGE], bar_sfull, bar_sfree, bar_pfull[2], bar_odone,
      bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ int n_union;
  __shared__ int never_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  const long long bh = blockIdx.y;
  const int b_idx = (int)(bh / prm.H), h_idx = (int)(bh % prm.H);
  const int qb0 = 2 * pair, qb1 = 2 * pair + 1;
  const bool has1 = qb1 < prm.nB;
  const int nW = (prm.nB + 31) >> 5;
  uint32_t* m0 = reinterpret_cast<uint32_t*>(sm + C::OFF_MASK);
  uint32_t* m1 = m0 + nW;
  float* sk_s = reinterpret_cast<float*>(m1 + nW);  // INT8: this head's K block scales

  // ---- prologue: barriers, kept-list bitmasks (validated), TMEM
  if (threadIdx.x == 0) {
    mbar_init(&bar_q, 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(&bar_sfull, 1);
    mbar_init(&bar_sfree, 128);
    for (int i = 0; i < 2; ++i) mbar_init(&bar_pfull[i], 128);
    mbar_init(&bar_odone, 1);
    mbar_init(&bar_drain, 1);
    abort_flag = 0;
    never_abort = 0;
    fence_barrier_init();
  }
  for (int w = threadIdx.x; w < 2 * nW; w += blockDim.x) m0[w] = 0u;
  if constexpr (I8)
    for (int jj = threadIdx.x; jj < prm.nB; jj += blockDim.x) sk_s[jj] = prm.sk[bh * prm.nB + jj];
  __syncthreads();
  {
    const int32_t* r0 = prm.idx + (bh * prm.nB + qb0) * (long long)prm.k;
    const int32_t* r1 = prm.idx + (bh * prm.nB + qb1) * (long long)prm.k;
    bool bad = false;
    for (int t = threadIdx.x; t < prm.k; t += blockDim.x) {
      const int j = r0[t];
      if (j < 0 || j >= prm.nB || (t > 0 && r0[t - 1] >= j)) bad = true;
      else atomicOr(&m0[j >> 5], 1u << (j & 31));
      if (has1) {
        const int j1 = r1[t];
        if (j1 < 0 || j1 >= prm.nB || (t > 0 && r1[t - 1] >= j1)) bad = true;
        else atomicOr(&m1[j1 >> 5], 1u << (j1 & 31));
      }
    }
    if (bad) report_error(-7);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    int cnt = 0;
    for (int w = lane; w < nW; w += 32) cnt += __popc(m0[w] | m1[w]);
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) n_union = cnt;
  }
  __syncthreads();
  const int n = n_union;
  const uint32_t tbase = tmem_slot;
  const uint32_t sQ = smem_u32(sm + C::OFF_Q);

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(&bar_q, C::Q_BYTES);
      for (int a = 0; a < C::NATOM; ++a)
        tma_load_4d(sm + C::OFF_Q + a * 128 * C::ATOM, &tmQ, &bar_q, a * C::ATOM / C::ESZ, qb0 * kBlock, h_idx, b_idx);
      UnionWalk uw;
      uw.init(m0, m1, nW);
      int j, fl, c = 0;
      while (uw.next(j, fl)) {
        const int s = c % C::NSTAGE;
        if (c >= C::NSTAGE && !mbar_wait(&bar_empty[s], ((c / C::NSTAGE) - 1) & 1, &abort_flag, prm.limit_ns)) {
          abort_flag = 1;
          report_error(-6);
          break;
        }
        mbar_arrive_expect_tx(&bar_full[s], 2 * C::KV_BYTES);
        for (int a = 0; a < C::NATOM; ++a) {
          tma_load_4d(sm + C::OFF_K + s * C::KV_BYTES + a * 64 * C::ATOM, &tmK, &bar_full[s], a * C::ATOM / C::ESZ,
                      j * kBlock, h_idx, b_idx);
          tma_load_4d(sm + C::OFF_V + s * C::KV_BYTES + a * 64 * C::ATOM, &tmV, &bar_full[s], a * C::ATOM / C::ESZ,
                      j * kBlock, h_idx, b_idx);
        }
        ++c;
      }
      // drain: every issued load lands before the CTA may exit
      mbar_wait(&bar_q, 0, &never_abort, prm.limit_ns);
      for (int cc = c - C::NSTAGE < 0 ? 0 : c - C::NSTAGE; cc < c; ++cc)
        mbar_wait(&bar_full[cc % C::NSTAGE], (cc / C::NSTAGE) & 1, &never_abort, prm.limit_ns);
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      bool ok = mbar_wait(&bar_q, 0, &abort_flag, prm.limit_ns);
      tc_fence_after();
      for (int c = 0; ok && c <= n; ++c) {
        if (c < n) {
          const int s = c % C::NSTAGE;
          ok = mbar_wait(&bar_full[s], (c / C::NSTAGE) & 1, &abort_flag, prm.limit_ns) &&
               mbar_wait(&bar_sfree, c & 1, &abort_flag, prm.limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sK = smem_u32(sm + C::OFF_K + s * C::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < C::ROWB / 32; ++kk) {
            const int a = (kk * 32) / C::ATOM, off = (kk * 32) % C::ATOM;
            const uint64_t ad = smem_desc(sQ + a * 128 * C::ATOM + off, 16, 8 * C::ATOM, C::SW_QKV);
            const uint64_t bd = smem_desc(sK + a * 64 * C::ATOM + off, 16, 8 * C::ATOM, C::SW_QKV);
            // INT8: accumulate onto the magic-number start the softmax warps wrote
            mma_ss<I8 ? KIND_I8 : KIND_F16>(tbase + C::S_COL, ad, bd, C::IDESC_S, (I8 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar_sfull);
        }
        if (c >= 1) {
          const int cp = c - 1, s = cp % C::NSTAGE, pb = cp & 1;
          ok = mbar_wait(&bar_pfull[pb], (cp >> 1) & 1, &abort_flag, prm.limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sV = smem_u32(sm + C::OFF_V + s * C::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < 64 / C::KEYS_PER_MMA; ++kk) {
            const uint64_t bd = smem_desc(sV + kk * C::KEYS_PER_MMA * C::ATOM, 64 * C::ATOM, 8 * C::ATOM, C::SW_QKV);
            mma_ts<I8 ? KIND_F8F6F4 : KIND_F16>(tbase + C::O_COL, tbase + C::P_COL + pb * C::P_COLS + kk * 8, bd,
                                                C::IDESC_PV, (cp > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar_odone);
          mma_commit(&bar_empty[s]);
        }
      }
      if (!ok) {
        abort_flag = 1;
        report_error(-6);
      }
      // drain: all issued MMAs complete before TMEM is released
      mma_commit(&bar_drain);
      mbar_wait(&bar_drain, 0, &never_abort, prm.limit_ns);
    }
  } else {
    // ================= softmax / correction / epilogue =================
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;           // tile row == TMEM lane
    const int half = r >> 6;
    const int qblk = half ? qb1 : qb0;
    const int t = qblk * kBlock + (r & 63);      // token index of this row
    const uint32_t lane_addr = tbase + ((uint32_t)(quarter * 32) << 16);
    float sq = 1.0f;
    if constexpr (I8) sq = prm.sq[bh * prm.nB + min(qblk, prm.nB - 1)];
    float m_run = -INFINITY, l_run = 0.f;
    // the S tile starts free (INT8: at the magic-number start value)
    if constexpr (I8) {
      uint32_t mg[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) mg[i] = kMagicBits;
      tmem_st32(lane_addr + C::S_COL, mg);
      tmem_st32(lane_addr + C::S_COL + 32, mg);
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(&bar_sfree);
    UnionWalk uw;
    uw.init(m0, m1, nW);
    bool ok = true;
    int j = 0, fl = 0;
    for (int c = 0; c < n; ++c) {
      uw.next(j, fl);
      const int bsel = c & 1;
      ok = mbar_wait(&bar_sfull, c & 1, &abort_flag, prm.limit_ns);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64];
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        tmem_ld32(lane_addr + C::S_COL, lo);
        tmem_ld32(lane_addr + C::S_COL + 32, hi);
        tmem_wait_ld();
      }
      // hand the S tile back at once (INT8: restarted at the magic value) so the
      // next S = QK^T runs on the tensor core while this block's softmax runs
      if constexpr (I8) {
        uint32_t mg[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) mg[i] = kMagicBits;
        tmem_st32(lane_addr + C::S_COL, mg);
        tmem_st32(lane_addr + C::S_COL + 32, mg);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&bar_sfree);
      const bool use = ((fl >> half) & 1) != 0;
      const int nvalid = (j == prm.nB - 1) ? (prm.L - j * kBlock) : kBlock;
      float sc = prm.scale_log2;
      if constexpr (I8) sc *= sq * sk_s[j];
      float m_new = m_run, alpha = 1.f, psum = 0.f;
      constexpr int PW = C::P_COLS;
      uint32_t pk[PW];
      if (use) {
        // block max (scores read as floats; INT8 ones carry the magic offset)
        float mx;
        if (nvalid == kBlock) {
          float t8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) t8[i] = __uint_as_float(sv[i]);
#pragma unroll
          for (int u = 8; u < 64; ++u) t8[u & 7] = fmaxf(t8[u & 7], __uint_as_float(sv[u]));
          mx = fmaxf(fmaxf(fmaxf(t8[0], t8[1]), fmaxf(t8[2], t8[3])), fmaxf(fmaxf(t8[4], t8[5]), fmaxf(t8[6], t8[7])));
        } else {
          mx = -INFINITY;
#pragma unroll
          for (int u = 0; u < 64; ++u)
            if (u < nvalid) mx = fmaxf(mx, __uint_as_float(sv[u]));
        }
        const float mblk = (I8 ? (mx - kMagic) : mx) * sc;
        m_new = fmaxf(m_run, mblk);
        alpha = (m_run == -INFINITY) ? 0.f : ex2f(m_run - m_new);
        // exponent argument x = s*sc - m (INT8: P lands on [0, 448] for the E4M3 cast)
        const float moff = I8 ? (m_new - kLog2_448) : m_new;
        const uint64_t sc2 = f2pack(sc, sc), nm2 = f2pack(-moff, -moff);
        const uint64_t mg2 = f2pack(-kMagic, -kMagic);
        uint64_t acc2[4] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f), f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
        const bool partial = nvalid < kBlock;
#pragma unroll
        for (int u = 0; u < 64; u += 2) {
          uint64_t s2 = f2pack(__uint_as_float(sv[u]), __uint_as_float(sv[u + 1]));
          if constexpr (I8) s2 = add2(s2, mg2);  // exact: the integer score as a float
          const uint64_t x2 = fma2(s2, sc2, nm2);
          float x0, x1;
          f2unpack(x2, x0, x1);
          sv[u] = __float_as_uint(ex2f(x0));
          sv[u + 1] = __float_as_uint(ex2f(x1));
        }
        if (partial) {
#pragma unroll
          for (int u = 0; u < 64; ++u)
            if (u >= nvalid) sv[u] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 64; u += 2) {
          const float p0 = __uint_as_float(sv[u]), p1 = __uint_as_float(sv[u + 1]);
          acc2[(u >> 1) & 3] = add2(acc2[(u >> 1) & 3], f2pack(p0, p1));
          if constexpr (I8) {
            const uint32_t e = e4m3x2(p0, p1);
            if ((u & 2) == 0) pk[u >> 2] = e;
            else pk[u >> 2] |= e << 16;
          } else {
            __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
            pk[u >> 1] = *reinterpret_cast<uint32_t*>(&hb);
          }
        }
        float a0, a1, a2, a3, b0, b1, b2, b3;
        f2unpack(acc2[0], a0, b0);
        f2unpack(acc2[1], a1, b1);
        f2unpack(acc2[2], a2, b2);
        f2unpack(acc2[3], a3, b3);
        psum = ((a0 + b0) + (a1 + b1)) + ((a2 + b2) + (a3 + b3));
      } else {
#pragma unroll
        for (int i = 0; i < PW; ++i) pk[i] = 0u;
      }
      if (c >= 1) {
        // PV of the previous block is complete: O may be rescaled and the P
        // buffer of block c-2 is free again
        ok = mbar_wait(&bar_odone, (c - 1) & 1, &abort_flag, prm.limit_ns);
        if (!ok) break;
        tc_fence_after();
        const bool need_rescale = use && m_run != -INFINITY && m_new > m_run;
        if (__any_sync(0xffffffffu, need_rescale)) {
          const float f = need_rescale ? alpha : 1.f;
#pragma unroll
          for (int cc = 0; cc < D; cc += 32) {
            uint32_t o[32];
            tmem_ld32(lane_addr + C::O_COL + cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(lane_addr + C::O_COL + cc, o);
          }
        }
      }
      // P of this block into its TMEM buffer: the A operand of PV
      if constexpr (I8) {
        tmem_st16(lane_addr + C::P_COL + bsel * C::P_COLS, pk);
      } else {
        tmem_st32(lane_addr + C::P_COL + bsel * C::P_COLS, *reinterpret_cast<uint32_t(*)[32]>(pk));
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_pfull[bsel]);
      if (use) {
        l_run = l_run * alpha + psum;
        m_run = m_new;
      }
    }
    if (!ok) {
      abort_flag = 1;
      report_error(-6);
    } else {
      // epilogue: wait for the last PV, normalise, store bf16 rows
      ok = n == 0 || mbar_wait(&bar_odone, (n - 1) & 1, &abort_flag, prm.limit_ns);
      if (!ok) {
        abort_flag = 1;
        report_error(-6);
      } else {
        tc_fence_after();
        const bool store = t < prm.L && (half == 0 || has1) && l_run > 0.f;
        const float inv_l = store ? 1.0f / l_run : 0.f;
        __nv_bfloat16* orow = prm.o + (long long)b_idx * prm.osB + (long long)h_idx * prm.osH + (long long)t * prm.osL;
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
          uint32_t o[32];
          tmem_ld32(lane_addr + C::O_COL + cc, o);
          tmem_wait_ld();
          if (store) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              float f0 = __uint_as_float(o[i]) * inv_l, f1 = __uint_as_float(o[i + 1]) * inv_l;
              if constexpr (I8) {
                f0 *= prm.sv[bh * D + cc + i];
                f1 *= prm.sv[bh * D + cc + i + 1];
              }
              __nv_bfloat162 hb = __floats2bfloat162_rn(f0, f1);
              w[i >> 1] = *reinterpret_cast<uint32_t*>(&hb);
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              *reinterpret_cast<uint4*>(orow + cc + 8 * q4) = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// A kernel that waits on a barrier nothing will ever complete, with a bound,
// then reports a timeout: exercises the failure path without hanging the GPU.
__global__ void wait_timeout_probe_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int never;
  if (threadIdx.x == 0) {
    never = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &never, limit_ns)) report_error(-6);
}

}  // namespace lx
