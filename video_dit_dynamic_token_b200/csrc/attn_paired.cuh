// Sparse attention over the kept key blocks (step a4), paired-S form: the
// kernel that INT8/FP8 calls run (measured 2-4 % faster there than the
// per-step form of attn.cuh, which BF16 calls run).
//
// "600倍加速，720p视频实时生成！单卡也能带的动14B模型", §动态稀疏量化注意力: only the
// activated attention tiles are computed and a chosen block stays dense
// inside; §高效推理算子: Q/K INT8 and V FP8.  "Run Wan2.2-A14B on One RTX 5090:
// 720p Video in 3.8s", §3 Dynamic sparse attention: the same in English.
//
// Tile: one CTA owns two adjacent 64-row query blocks (2p, 2p+1), run as two
// independent M=64 streams A and B in lockstep; two CTAs share an SM.  Step c
// computes query block 2p against its c-th kept key block and query block
// 2p+1 against ITS c-th kept key block, so every row works on one of its own
// kept blocks at every step and a CTA takes exactly k steps.  The two M=64
// accumulators of a step share TMEM columns: stream A in lanes 0-15 and
// stream B in lanes 16-31 of each 32-lane subpartition, so one warp's 32x32b
// TMEM load returns 16 rows of A and 16 rows of B.
//
// S is computed for two consecutive kept blocks of a stream at once (M=64,
// N=128 over the stacked blocks, one S buffer); P.V and the O rescale stay per
// 64-key block.  P is single-buffered and the softmax waits for P.V(c-1)
// before it writes P(c).
//
// Roles (6 warps): warp 0 = TMA producer (Q once; K blocks of both streams, a
// pair of steps at a time, into one stage, reused once that pair's S is
// complete; V blocks into a 2-stage ring), one thread; warp 1 = TMEM allocator
// + MMA issuer, a warp-wide loop whose waits are voted and whose MMAs one
// elected lane issues; warps 2..5 = softmax / correction /
// epilogue, one thread per (stream, row): thread t of warp w reads TMEM lane
// 32*(w%4) + t, i.e. row 16*(w%4) + t%16 of stream t/16.
//
// INT8/FP8 mode follows the P-quantisation protocol stated in attn.cuh; the
// kernel also has a BF16 form, which the library does not launch.
#pragma once
#include "attn.cuh"

namespace lx {

template <int D, bool I8>
struct AttnPairCfg {
  static constexpr int ESZ = I8 ? 1 : 2;                 // bytes per Q/K/V element
  static constexpr int ROWB = D * ESZ;                    // bytes per token row
  static constexpr int ATOM = ROWB >= 128 ? 128 : ROWB;   // swizzle atom width (128 or 64 bytes)
  static constexpr int NATOM = ROWB / ATOM;               // atom columns per row
  static constexpr int Q_BYTES = 128 * ROWB;              // rows 0-63: stream A, rows 64-127: stream B
  static constexpr int KV_BYTES = 64 * ROWB;              // one K (or V) block
  static constexpr int KPAIR_BYTES = 2 * KV_BYTES;        // one stream's two K blocks: [NATOM][128 rows][ATOM]
  static constexpr int VSTAGE = 2;                        // V ring (A and B blocks per stage)
  static constexpr int P_ROWB = 64 * ESZ;                 // P row: 64 keys
  static constexpr int P_BYTES = 64 * P_ROWB;             // P of one stream, K-major, swizzled
  static constexpr uint32_t SW_QKV = ATOM == 128 ? SW_128B : SW_64B;
  static constexpr uint32_t SW_P = P_ROWB == 128 ? SW_128B : SW_64B;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + 2 * KPAIR_BYTES;
  static constexpr int OFF_P = OFF_V + VSTAGE * 2 * KV_BYTES;
  static constexpr int OFF_IDX = OFF_P + 2 * P_BYTES;     // the two kept lists (2 x k int32) follow
  static constexpr int S_COL = 0;                         // TMEM: S of a step pair, cols [0, 128)
  static constexpr int O_COL = 128;                       // TMEM: O accumulator, D cols
  static constexpr uint32_t LANE_B = 16u << 16;           // TMEM address offset of stream B (lane 16)
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t IDESC_S =
      instr_desc(I8 ? IDESC_DS32 : IDESC_DF32, I8 ? IDESC_S8 : IDESC_BF16, I8 ? IDESC_S8 : IDESC_BF16, 0, 0, 64, 128);
  static constexpr uint32_t IDESC_PV =
      instr_desc(IDESC_DF32, I8 ? IDESC_E4M3 : IDESC_BF16, I8 ? IDESC_E4M3 : IDESC_BF16, 0, 1, 64, D);
  static constexpr int KEYS_PER_MMA = 32 / ESZ;           // 32 bytes of K per instruction
};

template <int D, bool I8>
__global__ void __launch_bounds__(192, I8 ? 2 : 1)
    sparse_attn_paired_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams prm) {
  using C = AttnPairCfg<D, I8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_q, bar_kfull, bar_vfull[C::VSTAGE],
      bar_vempty[C::VSTAGE], bar_sfull, bar_sfree, bar_pfull, bar_odone, bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ int never_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  const long long bh = blockIdx.y;
  const int b_idx = (int)(bh / prm.H), h_idx = (int)(bh % prm.H);
  const int qb0 = 2 * pair, qb1 = 2 * pair + 1;
  const bool has1 = qb1 < prm.nB;
  const int n = prm.k;  // steps: every stream walks exactly k kept blocks
  const int npairs = (n + 1) >> 1;  // S is computed for steps 2p and 2p+1 together
  int32_t* idx0 = reinterpret_cast<int32_t*>(sm + C::OFF_IDX);
  int32_t* idx1 = idx0 + n;

  // ---- prologue: barriers, the two kept lists (validated), TMEM
  if (threadIdx.x == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_kfull, 1);
    for (int s = 0; s < C::VSTAGE; ++s) {
      mbar_init(&bar_vfull[s], 1);
      mbar_init(&bar_vempty[s], 1);
    }
    mbar_init(&bar_sfull, 1);
    mbar_init(&bar_sfree, 128);
    mbar_init(&bar_pfull, 128);
    mbar_init(&bar_odone, 1);
    mbar_init(&bar_drain, 1);
    abort_flag = 0;
    never_abort = 0;
    fence_barrier_init();
  }
  {
    // an id out of range or out of order is reported; out-of-range ids are
    // replaced by 0 so that no load or scale lookup leaves its tensor
    const int32_t* r0 = prm.idx + (bh * prm.nB + qb0) * (long long)n;
    const int32_t* r1 = prm.idx + (bh * prm.nB + (has1 ? qb1 : qb0)) * (long long)n;
    bool bad = false;
    for (int t = threadIdx.x; t < n; t += blockDim.x) {
      int j0 = r0[t], j1 = r1[t];
      if (j0 < 0 || j0 >= prm.nB || (t > 0 && r0[t - 1] >= j0)) bad = true;
      if (j1 < 0 || j1 >= prm.nB || (t > 0 && r1[t - 1] >= j1)) bad = true;
      idx0[t] = (j0 < 0 || j0 >= prm.nB) ? 0 : j0;
      idx1[t] = (j1 < 0 || j1 >= prm.nB) ? 0 : j1;
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
      const uint32_t kv_tx = (has1 ? 2 : 1) * C::KV_BYTES;
      bool ok = true;
      int nk = 0, nv = 0;  // K pairs and V steps issued so far
      for (int c = 0; c < n; ++c) {
        if ((c & 1) == 0) {
          // K blocks of steps c and c+1 (both streams) into the pair stage,
          // once S of the previous pair has read it
          const int p = c >> 1;
          ok = p == 0 || mbar_wait(&bar_sfull, (p - 1) & 1, &abort_flag, prm.limit_ns);
          if (!ok) break;
          const int nb = (c + 1 < n) ? 2 : 1;
          mbar_arrive_expect_tx(&bar_kfull, (uint32_t)nb * kv_tx);
          for (int s = 0; s < (has1 ? 2 : 1); ++s) {
            const int32_t* ids = s ? idx1 : idx0;
            for (int b = 0; b < nb; ++b)
              for (int a = 0; a < C::NATOM; ++a)
                tma_load_4d(sm + C::OFF_K + s * C::KPAIR_BYTES + a * 128 * C::ATOM + b * 64 * C::ATOM, &tmK,
                            &bar_kfull, a * C::ATOM / C::ESZ, ids[c + b] * kBlock, h_idx, b_idx);
          }
          ++nk;
        }
        const int vs = c % C::VSTAGE;
        ok = c < C::VSTAGE || mbar_wait(&bar_vempty[vs], ((c / C::VSTAGE) - 1) & 1, &abort_flag, prm.limit_ns);
        if (!ok) break;
        const int j0 = idx0[c], j1 = idx1[c];
        uint8_t* sv = sm + C::OFF_V + vs * 2 * C::KV_BYTES;
        mbar_arrive_expect_tx(&bar_vfull[vs], kv_tx);
        for (int a = 0; a < C::NATOM; ++a) {
          tma_load_4d(sv + a * 64 * C::ATOM, &tmV, &bar_vfull[vs], a * C::ATOM / C::ESZ, j0 * kBlock, h_idx, b_idx);
          if (has1)
            tma_load_4d(sv + C::KV_BYTES + a * 64 * C::ATOM, &tmV, &bar_vfull[vs], a * C::ATOM / C::ESZ,
                        j1 * kBlock, h_idx, b_idx);
        }
        ++nv;
      }
      if (!ok) {
        abort_flag = 1;
        report_error(-6);
      }
      // drain: every issued load lands before the CTA may exit
      mbar_wait(&bar_q, 0, &never_abort, prm.limit_ns);
      if (nk > 0) mbar_wait(&bar_kfull, (nk - 1) & 1, &never_abort, prm.limit_ns);
      for (int cc = nv - C::VSTAGE < 0 ? 0 : nv - C::VSTAGE; cc < nv; ++cc)
        mbar_wait(&bar_vfull[cc % C::VSTAGE], (cc / C::VSTAGE) & 1, &never_abort, prm.limit_ns);
    }
  } else if (warp == 1) {
    // ================= MMA issuer (warp-wide loop, one elected lane issues) =================
    const bool leader = elect_one();
    {
      // Descriptors of stage 0 / stream A; a shared-memory descriptor's start
      // address sits in its low 14 bits (address >> 4, below 256 KB), so other
      // stages, streams and K steps are plain additions of (offset >> 4).
      const uint64_t dQ = smem_desc(sQ, 16, 8 * C::ATOM, C::SW_QKV);
      const uint64_t dK = smem_desc(smem_u32(sm + C::OFF_K), 16, 8 * C::ATOM, C::SW_QKV);
      const uint64_t dP = smem_desc(smem_u32(sm + C::OFF_P), 16, 8 * C::P_ROWB, C::SW_P);
      const uint64_t dV = smem_desc(smem_u32(sm + C::OFF_V), 64 * C::ATOM, 8 * C::ATOM, C::SW_QKV);
      bool ok = warp_wait(&bar_q, 0, &abort_flag, prm.limit_ns);
      tc_fence_after();
      // Iteration c issues S of pair p+1 (when c = 2p+1; pair 0 goes first)
      // and then P(c).V.  S of pair p+1 needs the softmax to have read both
      // halves of pair p's S, which it does at the start of step 2p+1.
      for (int c = -1; ok && c < n; ++c) {
        const int p = (c + 1) >> 1;  // the pair whose S is issued in this iteration
        if ((c & 1) != 0 && p < npairs) {  // c = -1, 1, 3, ...
          ok = warp_wait(&bar_kfull, p & 1, &abort_flag, prm.limit_ns) &&
               warp_wait(&bar_sfree, p & 1, &abort_flag, prm.limit_ns);
          if (!ok) break;
          tc_fence_after();
          if (leader) {
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            if (s == 1 && !has1) break;
#pragma unroll
            for (int kk = 0; kk < C::ROWB / 32; ++kk) {
              const int a = (kk * 32) / C::ATOM, off = (kk * 32) % C::ATOM;
              const uint64_t ad = dQ + (uint64_t)((a * 128 * C::ATOM + s * 64 * C::ATOM + off) >> 4);
              const uint64_t bd = dK + (uint64_t)((s * C::KPAIR_BYTES + a * 128 * C::ATOM + off) >> 4);
              // INT8: accumulate onto the magic-number start the softmax warps wrote
              mma_ss<I8 ? KIND_I8 : KIND_F16>(tbase + s * C::LANE_B + C::S_COL, ad, bd, C::IDESC_S,
                                              (I8 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(&bar_sfull);   // S complete: also frees the K pair stage
          }
          __syncwarp();
        }
        if (c >= 0) {
          const int vs = c % C::VSTAGE;
          ok = warp_wait(&bar_vfull[vs], (c / C::VSTAGE) & 1, &abort_flag, prm.limit_ns) &&
               warp_wait(&bar_pfull, c & 1, &abort_flag, prm.limit_ns);
          if (!ok) break;
          tc_fence_after();
          if (leader) {
          const uint64_t dVs = dV + (uint64_t)((vs * 2 * C::KV_BYTES) >> 4);
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            if (s == 1 && !has1) break;
#pragma unroll
            for (int kk = 0; kk < 64 / C::KEYS_PER_MMA; ++kk) {
              const uint64_t ad = dP + (uint64_t)((s * C::P_BYTES + kk * 32) >> 4);
              const uint64_t bd = dVs + (uint64_t)((s * C::KV_BYTES + kk * C::KEYS_PER_MMA * C::ATOM) >> 4);
              mma_ss<I8 ? KIND_F8F6F4 : KIND_F16>(tbase + s * C::LANE_B + C::O_COL, ad, bd, C::IDESC_PV,
                                                  (c > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(&bar_odone);
          mma_commit(&bar_vempty[vs]);
          }
          __syncwarp();
        }
      }
      if (!ok && leader) {
        abort_flag = 1;
        report_error(-6);
      }
      // drain: all issued MMAs complete before TMEM is released
      if (leader) {
        mma_commit(&bar_drain);
        mbar_wait(&bar_drain, 0, &never_abort, prm.limit_ns);
      }
      __syncwarp();
    }
  } else {
    // ================= softmax / correction / epilogue =================
    const int quarter = warp & 3;
    const int stream = lane >> 4;
    const int row = quarter * 16 + (lane & 15);   // row within this stream's query block
    const int qblk = stream ? qb1 : qb0;
    const bool valid = stream == 0 || has1;
    const int t = qblk * kBlock + row;            // token index of this row
    const uint32_t lane_addr = tbase + ((uint32_t)(quarter * 32) << 16);
    const int32_t* my_idx = stream ? idx1 : idx0;
    const float* sk_row = prm.sk + bh * prm.nB;
    float sq = 1.0f;
    if constexpr (I8) sq = prm.sq[bh * prm.nB + min(qblk, prm.nB - 1)];
    float m_run = -INFINITY, l_run = 0.f;
    // this thread's row of its stream's P tile (K-major, swizzled)
    uint8_t* prow = sm + C::OFF_P + stream * C::P_BYTES;
    // the S columns start free (INT8: at the magic-number start value)
    if constexpr (I8) {
      uint32_t mg[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) mg[i] = kMagicBits;
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_st32(lane_addr + C::S_COL + 32 * q, mg);
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(&bar_sfree);
    bool ok = true;
    int j_next = n > 0 ? my_idx[0] : 0;
    float sk_next = (I8 && n > 0) ? __ldg(sk_row + j_next) : 1.f;
    for (int c = 0; c < n; ++c) {
      const int j = j_next;
      const float skj = sk_next;
      if (c + 1 < n) {  // the next step's block and K scale, fetched a step ahead
        j_next = my_idx[c + 1];
        if constexpr (I8) sk_next = __ldg(sk_row + j_next);
      }
      const int half = c & 1;  // which 64 columns of the pair's S
      const uint32_t s_addr = lane_addr + C::S_COL + 64 * half;
      if (half == 0) {
        ok = mbar_wait(&bar_sfull, (c >> 1) & 1, &abort_flag, prm.limit_ns);
        if (!ok) break;
      }
      tc_fence_after();
      uint32_t sv[64];
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        tmem_ld32(s_addr, lo);
        tmem_ld32(s_addr + 32, hi);
        tmem_wait_ld();
      }
      // INT8: restart these columns at the magic value; after the second half
      // of the pair the S columns go back to the MMA thread at once, so the
      // next pair's S = QK^T runs while this block's softmax runs
      if constexpr (I8) {
        uint32_t mg[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) mg[i] = kMagicBits;
        tmem_st32(s_addr, mg);
        tmem_st32(s_addr + 32, mg);
        tmem_wait_st();
      }
      if (half == 1) {
        tc_fence_before();
        mbar_arrive(&bar_sfree);
      }
      const int nvalid = (j == prm.nB - 1) ? (prm.L - j * kBlock) : kBlock;
      float sc = prm.scale_log2;
      if constexpr (I8) sc *= sq * skj;
      float m_new = m_run, alpha = 1.f, psum = 0.f;
      constexpr int PW = C::P_ROWB / 4;
      uint32_t pk[PW];
      if (valid) {
        // block max (scores read as floats; INT8 ones carry the magic offset)
        float mx;
        if (nvalid == kBlock) {
          // eight chains of three-input maxima, then a three-level fold
          const float* f = reinterpret_cast<const float*>(sv);
          float t8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float a = fmax3(f[i], f[i + 8], f[i + 16]);
            a = fmax3(a, f[i + 24], f[i + 32]);
            a = fmax3(a, f[i + 40], f[i + 48]);
            t8[i] = fmaxf(a, f[i + 56]);
          }
          mx = fmaxf(fmax3(t8[0], t8[1], t8[2]), fmax3(t8[3], t8[4], fmax3(t8[5], t8[6], t8[7])));
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
            if ((u & 2) == 0)
              pk[u >> 2] = e4m3x4(p0, p1, __uint_as_float(sv[u + 2]), __uint_as_float(sv[u + 3]));
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
        // the previous block's P.V is complete: O may be rescaled and the P
        // tiles may be overwritten
        ok = mbar_wait(&bar_odone, (c - 1) & 1, &abort_flag, prm.limit_ns);
        if (!ok) break;
        tc_fence_after();
        const bool need_rescale = valid && m_run != -INFINITY && m_new > m_run;
        if (__any_sync(0xffffffffu, need_rescale)) {
          const float f = need_rescale ? alpha : 1.f;
          const uint64_t f2 = f2pack(f, f);
#pragma unroll
          for (int cc = 0; cc < D; cc += 64) {   // two 32-column loads in flight per round trip
            uint32_t o[2][32];
            tmem_ld32(lane_addr + C::O_COL + cc, o[0]);
            if (cc + 32 < D) tmem_ld32(lane_addr + C::O_COL + cc + 32, o[1]);
            tmem_wait_ld();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (cc + 32 * hh < D) {
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                  float a, b;
                  f2unpack(mul2(f2pack(__uint_as_float(o[hh][i]), __uint_as_float(o[hh][i + 1])), f2), a, b);
                  o[hh][i] = __float_as_uint(a);
                  o[hh][i + 1] = __float_as_uint(b);
                }
                tmem_st32(lane_addr + C::O_COL + cc + 32 * hh, o[hh]);
              }
            }
          }
          tmem_wait_st();
        }
      }
      // P row into shared memory: the A operand of this stream's P.V
#pragma unroll
      for (int ch = 0; ch < C::P_ROWB / 16; ++ch)
        *reinterpret_cast<uint4*>(prow + swz_offset(row, ch, C::P_ROWB)) =
            make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bar_pfull);
      if (valid) {
        l_run = l_run * alpha + psum;
        m_run = m_new;
      }
    }
    if (!ok) {
      abort_flag = 1;
      report_error(-6);
    } else {
      // epilogue: wait for the last P.V, normalise, store bf16 rows
      ok = n == 0 || mbar_wait(&bar_odone, (n - 1) & 1, &abort_flag, prm.limit_ns);
      if (!ok) {
        abort_flag = 1;
        report_error(-6);
      } else {
        tc_fence_after();
        const bool store = valid && t < prm.L && l_run > 0.f;
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

}  // namespace lx
