// C-ABI host library: argument checks, TMA tensor maps, launches.
// The whole library is this one translation unit (kernels come in as headers).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "lx_sparse_attn.h"
#include "ptx.cuh"
#include "planner.cuh"
#include "quant.cuh"
#include "ulysses.cuh"
#include "nvfp4.cuh"
#include "attn.cuh"
#include "attn_paired.cuh"

namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // bound on every device-side wait
constexpr int64_t kMaxPlannerNB = 2176;  // selection: 8 score rows of nB fp32 in shared memory, 17 chunks of 128
static_assert(kMaxPlannerNB <= 128 * lx::kMaxChunks, "selection chunk registers too few for the longest row");

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t n_blocks(int64_t L) { return (L + LX_BLOCK - 1) / LX_BLOCK; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline int64_t keep_count(int64_t nB, double keep) {
  int64_t k = (int64_t)std::ceil(keep * (double)nB - 1e-6);
  return k < 1 ? 1 : (k > nB ? nB : k);
}

lx_status check_bhld(const lx_bhld* t) {
  if (!t || !t->data) return LX_ERR_INVALID;
  if (t->B < 1 || t->H < 1 || t->L < 1) return LX_ERR_INVALID;
  if (t->D != 64 && t->D != 128) return LX_ERR_UNSUPPORTED;
  if (t->sL < t->D || t->sH < 1 || t->sB < 1) return LX_ERR_INVALID;
  if (t->L > (int64_t)1 << 30 || t->B * t->H > (int64_t)1 << 30) return LX_ERR_UNSUPPORTED;
  if (!al16(t->data) || (t->sL * 2) % 16 || (t->sH * 2) % 16 || (t->sB * 2) % 16) return LX_ERR_ALIGN;
  return LX_OK;
}

inline bool same_shape(const lx_bhld* a, const lx_bhld* b) {
  return a->B == b->B && a->H == b->H && a->L == b->L && a->D == b->D;
}

inline lx::BhldView view(const lx_bhld* t) {
  return lx::BhldView{reinterpret_cast<const __nv_bfloat16*>(t->data), t->sB, t->sH, t->sL};
}

lx_status check_plan(const lx_plan* p, const lx_bhld* shape) {
  if (!p || !p->idx || !al16(p->idx)) return LX_ERR_INVALID;
  const int64_t nB = n_blocks(shape->L);
  if (p->B != shape->B || p->H != shape->H || p->L != shape->L || p->nB != nB || p->block != LX_BLOCK)
    return LX_ERR_INVALID;
  if (p->k < 1 || p->k > nB) return LX_ERR_INVALID;
  return LX_OK;
}

// Persistent 128-thread grid of the V quantiser: four CTAs per SM, each over a
// contiguous range of `per` units.
bool persistent_grid(long long units, long long* ctas, long long* per) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms < 1)
    return false;
  const long long want = 4LL * sms;
  *per = (units + want - 1) / want;
  *ctas = (units + *per - 1) / *per;
  return true;
}

// Score workspace of lx_score_topk: fp32 [B*H, nB, ldS], rows padded to a
// multiple of 32 floats so that each starts on a 128-byte boundary.
inline int64_t score_ld(int64_t nB) { return (nB + 31) / 32 * 32; }
inline size_t score_ws_bytes(int64_t BH, int64_t nB) {
  return align256(sizeof(float) * (size_t)(BH * nB * score_ld(nB)));
}

inline lx_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? LX_OK : LX_ERR_CUDA;
}

// ---------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 4-D map over [B,H,L,D] (innermost first: D, L, H, B), strides in elements.
bool make_map(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int esz, int64_t B, int64_t H, int64_t L,
              int64_t D, int64_t sB, int64_t sH, int64_t sL, int box_inner, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)H, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)(sL * esz), (cuuint64_t)(sH * esz), (cuuint64_t)(sB * esz)};
  const cuuint32_t box[4] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  const int inner_bytes = box_inner * esz;
  const CUtensorMapSwizzle sw = inner_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return fn(m, dt, 4, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- launchers
template <int D>
lx_status launch_qk_pass(const lx_bhld* Q, const lx_bhld* K, float* mq, float* mk, int8_t* qc, float* qs, int8_t* kc,
                         float* ks, cudaStream_t s, const lx::ProParams* pro = nullptr) {
  const int64_t nB = n_blocks(Q->L);
  dim3 grid((unsigned)(Q->B * Q->H * nB), 2);
  const int H = (int)Q->H, L = (int)Q->L;
  const lx::ProParams pp = pro ? *pro : lx::ProParams{};
  const lx::BhldView vq = view(Q), vk = view(K);
  if (pro) {
    if (qc)
      lx::qk_block_pass_kernel<D, true, true, true><<<grid, 128, 0, s>>>(vq, vk, mq, mk, qc, kc, qs, ks, H, L, (int)nB, pp);
    else
      lx::qk_block_pass_kernel<D, true, false, true><<<grid, 128, 0, s>>>(vq, vk, mq, mk, qc, kc, qs, ks, H, L, (int)nB, pp);
  } else if (mq && qc) {
    lx::qk_block_pass_kernel<D, true, true, false><<<grid, 128, 0, s>>>(vq, vk, mq, mk, qc, kc, qs, ks, H, L, (int)nB, pp);
  } else if (mq) {
    lx::qk_block_pass_kernel<D, true, false, false><<<grid, 128, 0, s>>>(vq, vk, mq, mk, qc, kc, qs, ks, H, L, (int)nB, pp);
  } else {
    lx::qk_block_pass_kernel<D, false, true, false><<<grid, 128, 0, s>>>(vq, vk, mq, mk, qc, kc, qs, ks, H, L, (int)nB, pp);
  }
  return launch_status();
}

// Scores of BH heads: tf32 x3 tensor-core GEMM, one 128 x 128 tile per CTA;
// mq, mk, scores point at the first of the BH heads.
template <int D>
lx_status launch_score_gemm(const float* mq, const float* mk, int64_t BH, int64_t nB, float* scores, cudaStream_t s) {
  CUtensorMap tq, tk;
  const auto f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (!make_map(&tq, mq, f32, 4, 1, BH, nB, D, BH * nB * D, nB * D, D, lx::kSgK, lx::kSgM) ||
      !make_map(&tk, mk, f32, 4, 1, BH, nB, D, BH * nB * D, nB * D, D, lx::kSgK, lx::kSgN))
    return LX_ERR_CUDA;
  const size_t gsmem = 1024 + lx::kSgSmem;
  if (cudaFuncSetAttribute(lx::score_gemm_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsmem) !=
      cudaSuccess)
    return LX_ERR_CUDA;
  dim3 ggrid((unsigned)((nB + lx::kSgM - 1) / lx::kSgM), (unsigned)((nB + lx::kSgN - 1) / lx::kSgN), (unsigned)BH);
  const int ldS = (int)score_ld(nB);
  lx::score_gemm_kernel<D><<<ggrid, 128, gsmem, s>>>(tq, tk, scores, (int)nB, ldS, kWaitLimitNs);
  return launch_status();
}

// Top-k selection of BH heads: 8 score rows per CTA, one warp per row; the
// pointers are those of the first of the BH heads (mask may be NULL).
lx_status launch_select(const float* scores, int64_t BH, int64_t nB, int64_t k, int32_t* idx, uint32_t* mask,
                        cudaStream_t s) {
  const int ldS = (int)score_ld(nB);
  const size_t smem = sizeof(float) * ((size_t)lx::kScoreRows * ldS +
                                       lx::kScoreWarps * (lx::kBuckets + 2 * lx::kCandCap + ldS / 32));
  if (smem > 227 * 1024) return LX_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(lx::select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LX_ERR_CUDA;
  dim3 grid((unsigned)((nB + lx::kScoreRows - 1) / lx::kScoreRows), (unsigned)BH);
  lx::select_topk_kernel<<<grid, 32 * lx::kScoreWarps, smem, s>>>(scores, (int)nB, (int)k, idx, mask, ldS,
                                                                   kWaitLimitNs);
  return launch_status();
}

template <int D>
lx_status launch_score(const float* mq, const float* mk, int64_t BH, int64_t nB, int64_t k, float* scores,
                       lx_plan* plan, cudaStream_t s) {
  lx_status st = launch_score_gemm<D>(mq, mk, BH, nB, scores, s);
  if (st != LX_OK) return st;
  return launch_select(scores, BH, nB, k, plan->idx, plan->mask, s);
}

template <int D, bool MEANS>
void launch_smooth(const lx_bhld* Q, const lx_bhld* K, const float* km, float* mq, float* mk, int8_t* qc, float* qs,
                   int8_t* kc, float* ks, cudaStream_t s) {
  const int64_t nB = n_blocks(Q->L);
  dim3 grid((unsigned)(Q->B * Q->H * nB), 2);
  lx::qk_block_pass_kernel<D, MEANS, true, false, true><<<grid, 128, 0, s>>>(
      view(Q), view(K), mq, mk, qc, kc, qs, ks, (int)Q->H, (int)Q->L, (int)nB, lx::ProParams{}, km);
}
template <int D>
lx_status launch_quant_v(const lx_bhld* V, uint8_t* vc, float* vs, uint32_t* amax, cudaStream_t s) {
  const int64_t BH = V->B * V->H, nB = n_blocks(V->L);
  const int nSpan = (int)((V->L + lx::kVSpan - 1) / lx::kVSpan);
  if (cudaMemsetAsync(amax, 0, sizeof(uint32_t) * BH * D, s) != cudaSuccess) return LX_ERR_CUDA;
  lx::v_absmax_kernel<D><<<(unsigned)(BH * nSpan), 128, 0, s>>>(view(V), amax, (int)V->H, (int)V->L, nSpan);
  if (cudaGetLastError() != cudaSuccess) return LX_ERR_CUDA;
  long long ctas = 0, per = 0;
  if (!persistent_grid(BH * nB, &ctas, &per)) return LX_ERR_CUDA;
  lx::v_quant_kernel<D><<<(unsigned)ctas, 128, 0, s>>>(view(V), amax, vc, vs, (int)V->H, (int)V->L, (int)nB,
                                                       (long long)(BH * nB), per);
  return launch_status();
}

// Kernel arguments shared by both attention kernels.
template <int D>
lx::AttnParams attn_params(const lx_plan* plan, const lx_bhld* O, const float* qs, const float* ks, const float* vs) {
  lx::AttnParams p;
  p.idx = plan->idx;
  p.k = (int)plan->k;
  p.nB = (int)plan->nB;
  p.L = (int)plan->L;
  p.H = (int)plan->H;
  p.o = reinterpret_cast<__nv_bfloat16*>(O->data);
  p.osB = O->sB;
  p.osH = O->sH;
  p.osL = O->sL;
  p.sq = qs;
  p.sk = ks;
  p.sv = vs;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  p.limit_ns = kWaitLimitNs;
  return p;
}

// one CTA per (pair of query blocks, b*h), head-major so that a head's K/V stays in L2
inline dim3 attn_grid(const lx_plan* plan) {
  return dim3((unsigned)((plan->nB + 1) / 2), (unsigned)(plan->B * plan->H));
}

// INT8/FP8 attention: the paired-S kernel (attn_paired.cuh)
template <int D>
lx_status launch_attn_paired(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const lx_plan* plan,
                             const lx_bhld* O, const float* qs, const float* ks, const float* vs, cudaStream_t s) {
  using C = lx::AttnPairCfg<D, true>;
  // the two kept lists follow the tiles
  const size_t smem = 1024 + C::OFF_IDX + 2 * sizeof(int32_t) * (size_t)plan->k;
  if (smem > 227 * 1024) return LX_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(lx::sparse_attn_paired_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return LX_ERR_CUDA;
  lx::sparse_attn_paired_kernel<D, true><<<attn_grid(plan), 192, smem, s>>>(mq, mk, mv,
                                                                           attn_params<D>(plan, O, qs, ks, vs));
  return launch_status();
}

// BF16 attention: the per-step kernel (attn.cuh)
template <int D, bool I8>
lx_status launch_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const lx_plan* plan,
                      const lx_bhld* O, const float* qs, const float* ks, const float* vs, cudaStream_t s) {
  using C = lx::AttnCfg<D, I8>;
  // the two kept lists and their K scales follow the tiles
  const size_t smem = 1024 + C::OFF_IDX + 16 * (size_t)plan->k;
  if (smem > 227 * 1024) return LX_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(lx::sparse_attn_kernel<D, I8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LX_ERR_CUDA;
  lx::sparse_attn_kernel<D, I8><<<attn_grid(plan), C::THREADS, smem, s>>>(mq, mk, mv,
                                                                          attn_params<D>(plan, O, qs, ks, vs));
  return launch_status();
}

template <int D>
lx_status attn_bf16_impl(const lx_bhld* Q, const lx_bhld* K, const lx_bhld* V, const lx_plan* plan, const lx_bhld* O,
                         cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&mq, Q->data, dt, 2, Q->B, Q->H, Q->L, D, Q->sB, Q->sH, Q->sL, 64, 128) ||
      !make_map(&mk, K->data, dt, 2, K->B, K->H, K->L, D, K->sB, K->sH, K->sL, 64, 64) ||
      !make_map(&mv, V->data, dt, 2, V->B, V->H, V->L, D, V->sB, V->sH, V->sL, 64, 64))
    return LX_ERR_CUDA;
  return launch_attn<D, false>(mq, mk, mv, plan, O, nullptr, nullptr, nullptr, s);
}

template <int D>
lx_status attn_i8_impl(const int8_t* qc, const float* qs, const int8_t* kc, const float* ks, const uint8_t* vc,
                       const float* vs, const lx_plan* plan, const lx_bhld* O, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const int64_t B = O->B, H = O->H, L = O->L;
  const int64_t sL = D, sH = L * D, sB = H * L * D;
  const auto dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  if (!make_map(&mq, qc, dt, 1, B, H, L, D, sB, sH, sL, D, 128) ||
      !make_map(&mk, kc, dt, 1, B, H, L, D, sB, sH, sL, D, 64) ||
      !make_map(&mv, vc, dt, 1, B, H, L, D, sB, sH, sL, D, 64))
    return LX_ERR_CUDA;
  return launch_attn_paired<D>(mq, mk, mv, plan, O, qs, ks, vs, s);
}

struct FwdWs {
  size_t qc, kc, vc, qs, ks, vs, amax, total;
};
FwdWs fwd_layout(const lx_bhld* Q) {
  FwdWs w;
  const size_t codes = (size_t)(Q->B * Q->H * Q->L * Q->D);
  const size_t bsc = sizeof(float) * (size_t)(Q->B * Q->H * n_blocks(Q->L));
  const size_t csc = sizeof(float) * (size_t)(Q->B * Q->H * Q->D);
  w.qc = 0;
  w.kc = w.qc + align256(codes);
  w.vc = w.kc + align256(codes);
  w.qs = w.vc + align256(codes);
  w.ks = w.qs + align256(bsc);
  w.vs = w.ks + align256(bsc);
  w.amax = w.vs + align256(csc);
  w.total = w.amax + align256(csc);
  return w;
}

}  // namespace

// ====================================================================== C ABI
// Light-Ulysses launch helper and the NVFP4 code map (the entries are below, in the C block)
namespace {
lx::BhldRW rw(const lx_bhld* t) {
  return lx::BhldRW{reinterpret_cast<__nv_bfloat16*>(t->data), t->sB, t->sH, t->sL};
}
template <int MODE>
lx_status launch_ulysses(lx::UlyssesArgs a, int64_t D, cudaStream_t s) {
  if (a.rows == 0) return LX_OK;
  // blockIdx.y: the (destination, batch, head) slices; blockIdx.x: rows of one slice
  const long long slices = (long long)a.N * a.B * a.Hc;
  const long long slice_rows = (long long)a.Lr * ((MODE == lx::kPackQKV || MODE == lx::kUnpackQKV) ? 3 : 1);
  const long long per_block = (256 / (D / 8)) * (long long)lx::kUlyPasses;  // rows per CTA
  if (slices > 65535 || slice_rows > (1LL << 30)) return LX_ERR_UNSUPPORTED;
  dim3 grid((unsigned)((slice_rows + per_block - 1) / per_block), (unsigned)slices);
  if (D == 128)
    lx::ulysses_rows_kernel<128, MODE><<<grid, 256, 0, s>>>(a);
  else
    lx::ulysses_rows_kernel<64, MODE><<<grid, 256, 0, s>>>(a);
  return launch_status();
}

// 2-D byte map over NVFP4 codes [rows][K/2] (innermost first), 128-byte swizzle,
// box of 128 bytes x box_rows rows; rows past the end read as zero.
bool make_map_codes(CUtensorMap* m, const void* ptr, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  const cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

const char* lx_status_string(lx_status st) {
  switch (st) {
    case LX_OK: return "ok";
    case LX_ERR_INVALID: return "invalid argument";
    case LX_ERR_UNSUPPORTED: return "unsupported shape";
    case LX_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
    case LX_ERR_WORKSPACE: return "workspace missing or too small";
    case LX_ERR_CUDA: return "CUDA error";
    case LX_ERR_TIMEOUT: return "device wait timed out";
    case LX_ERR_PLAN: return "malformed plan or non-finite scores";
  }
  return "unknown status";
}

lx_status lx_plan_size(int64_t B, int64_t H, int64_t L, int64_t D, double keep, int64_t* k, size_t* idx_bytes,
                       size_t* mask_bytes, size_t* ws_bytes) {
  if (B < 1 || H < 1 || L < 1 || !(keep > 0.0 && keep <= 1.0)) return LX_ERR_INVALID;
  if (D != 64 && D != 128) return LX_ERR_UNSUPPORTED;
  const int64_t nB = n_blocks(L), kk = keep_count(nB, keep);
  if (k) *k = kk;
  if (idx_bytes) *idx_bytes = sizeof(int32_t) * (size_t)(B * H * nB * kk);
  if (mask_bytes) *mask_bytes = sizeof(uint32_t) * (size_t)(B * H * nB * ((nB + 31) / 32));
  if (ws_bytes) *ws_bytes = 2 * align256(sizeof(float) * (size_t)(B * H * nB * D)) + score_ws_bytes(B * H, nB);
  return LX_OK;
}

lx_status lx_pool_means(const lx_bhld* Q, const lx_bhld* K, float* mq, float* mk, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK) return st;
  if (!same_shape(Q, K) || !mq || !mk) return LX_ERR_INVALID;
  if (!al16(mq) || !al16(mk)) return LX_ERR_ALIGN;
  return Q->D == 128 ? launch_qk_pass<128>(Q, K, mq, mk, nullptr, nullptr, nullptr, nullptr, stream)
                     : launch_qk_pass<64>(Q, K, mq, mk, nullptr, nullptr, nullptr, nullptr, stream);
}

lx_status lx_score_topk(const float* mq, const float* mk, int64_t B, int64_t H, int64_t L, int64_t D, double keep,
                        lx_plan* plan, void* ws, size_t ws_bytes, cudaStream_t stream) {
  int64_t k = 0;
  lx_status st = lx_plan_size(B, H, L, D, keep, &k, nullptr, nullptr, nullptr);
  if (st != LX_OK) return st;
  if (!mq || !mk || !plan || !plan->idx) return LX_ERR_INVALID;
  if (!al16(mq) || !al16(mk) || !al16(plan->idx) || (plan->mask && !al16(plan->mask))) return LX_ERR_ALIGN;
  const int64_t nB = n_blocks(L);
  if (nB > kMaxPlannerNB) return LX_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < score_ws_bytes(B * H, nB)) return LX_ERR_WORKSPACE;
  if (!al16(ws)) return LX_ERR_ALIGN;
  plan->B = B;
  plan->H = H;
  plan->L = L;
  plan->nB = nB;
  plan->k = k;
  plan->block = LX_BLOCK;
  float* scores = reinterpret_cast<float*>(ws);
  return D == 128 ? launch_score<128>(mq, mk, B * H, nB, k, scores, plan, stream)
                  : launch_score<64>(mq, mk, B * H, nB, k, scores, plan, stream);
}

lx_status lx_sparse_attn_plan(const lx_bhld* Q, const lx_bhld* K, double keep, lx_plan* plan, void* ws,
                              size_t ws_bytes, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK) return st;
  if (!same_shape(Q, K) || !plan) return LX_ERR_INVALID;
  size_t need = 0;
  if ((st = lx_plan_size(Q->B, Q->H, Q->L, Q->D, keep, nullptr, nullptr, nullptr, &need)) != LX_OK) return st;
  if (!ws || ws_bytes < need) return LX_ERR_WORKSPACE;
  if (!al16(ws)) return LX_ERR_ALIGN;
  if (n_blocks(Q->L) > kMaxPlannerNB) return LX_ERR_UNSUPPORTED;
  // workspace: [block means of Q | block means of K | scores], 256-byte aligned
  const size_t means = align256(sizeof(float) * (size_t)(Q->B * Q->H * n_blocks(Q->L) * Q->D));
  float* mq = reinterpret_cast<float*>(ws);
  float* mk = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + means);
  char* sc = reinterpret_cast<char*>(ws) + 2 * means;
  if ((st = lx_pool_means(Q, K, mq, mk, stream)) != LX_OK) return st;
  return lx_score_topk(mq, mk, Q->B, Q->H, Q->L, Q->D, keep, plan, sc, need - 2 * means, stream);
}

lx_status lx_quantize_qk(const lx_bhld* Q, const lx_bhld* K, int8_t* qc, float* qs, int8_t* kc, float* ks,
                         cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK) return st;
  if (!same_shape(Q, K) || !qc || !qs || !kc || !ks) return LX_ERR_INVALID;
  if (!al16(qc) || !al16(kc) || !al16(qs) || !al16(ks)) return LX_ERR_ALIGN;
  return Q->D == 128 ? launch_qk_pass<128>(Q, K, nullptr, nullptr, qc, qs, kc, ks, stream)
                     : launch_qk_pass<64>(Q, K, nullptr, nullptr, qc, qs, kc, ks, stream);
}

lx_status lx_pool_quantize_qk(const lx_bhld* Q, const lx_bhld* K, float* mq, float* mk, int8_t* qc, float* qs,
                              int8_t* kc, float* ks, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK) return st;
  if (!same_shape(Q, K) || !mq || !mk || !qc || !qs || !kc || !ks) return LX_ERR_INVALID;
  if (!al16(mq) || !al16(mk) || !al16(qc) || !al16(kc) || !al16(qs) || !al16(ks)) return LX_ERR_ALIGN;
  return Q->D == 128 ? launch_qk_pass<128>(Q, K, mq, mk, qc, qs, kc, ks, stream)
                     : launch_qk_pass<64>(Q, K, mq, mk, qc, qs, kc, ks, stream);
}

// ---------------------------------------------------------------- prologue (3D RoPE + RMSNorm)
namespace {
lx_status check_rope(const lx_rope3d* r, int64_t D) {
  if (!r) return LX_ERR_INVALID;
  if (D != 64 && D != 128) return LX_ERR_UNSUPPORTED;
  if (r->T < 1 || r->Hh < 1 || r->W < 1 || r->T * r->Hh * r->W > (int64_t)1 << 30) return LX_ERR_INVALID;
  if (r->dt < 0 || r->dh < 0 || r->dw < 0 || (r->dt | r->dh | r->dw) & 1 || r->dt + r->dh + r->dw != D)
    return LX_ERR_INVALID;
  if (!(r->theta > 0.0) || !std::isfinite(r->theta)) return LX_ERR_INVALID;
  return LX_OK;
}
int64_t rope_entries(const lx_rope3d* r) { return r->T * (r->dt / 2) + r->Hh * (r->dh / 2) + r->W * (r->dw / 2); }
}  // namespace

lx_status lx_rope3d_table_size(const lx_rope3d* rope, int64_t D, size_t* bytes) {
  lx_status st = check_rope(rope, D);
  if (st != LX_OK) return st;
  if (!bytes) return LX_ERR_INVALID;
  *bytes = sizeof(float) * 2 * (size_t)rope_entries(rope);
  return LX_OK;
}

lx_status lx_rope3d_table(const lx_rope3d* rope, int64_t D, float* table, cudaStream_t stream) {
  lx_status st = check_rope(rope, D);
  if (st != LX_OK) return st;
  if (!table) return LX_ERR_INVALID;
  if (!al16(table)) return LX_ERR_ALIGN;
  const int64_t n = rope_entries(rope);
  if (n == 0) return LX_OK;
  const unsigned blocks = (unsigned)std::min<int64_t>((n + 255) / 256, 1024);
  lx::rope3d_table_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<float2*>(table), (int)rope->T, (int)rope->Hh,
                                                       (int)rope->W, rope->dt / 2, rope->dh / 2, rope->dw / 2,
                                                       rope->theta);
  return launch_status();
}

lx_status lx_qk_prologue(const lx_bhld* Q, const lx_bhld* K, const float* wq, const float* wk, float eps,
                         const lx_rope3d* rope, const float* table, const lx_bhld* Yq, const lx_bhld* Yk, float* mq,
                         float* mk, int8_t* qc, float* qs, int8_t* kc, float* ks, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK) return st;
  if (!same_shape(Q, K)) return LX_ERR_INVALID;
  if ((st = check_rope(rope, Q->D)) != LX_OK) return st;
  if (Q->L > rope->T * rope->Hh * rope->W) return LX_ERR_INVALID;
  if (!wq || !wk || !table || !mq || !mk || !(eps >= 0.f) || !std::isfinite(eps)) return LX_ERR_INVALID;
  if ((qc == nullptr) != (kc == nullptr) || (qc == nullptr) != (qs == nullptr) || (qs == nullptr) != (ks == nullptr))
    return LX_ERR_INVALID;
  if ((Yq == nullptr) != (Yk == nullptr)) return LX_ERR_INVALID;
  if (Yq) {
    if ((st = check_bhld(Yq)) != LX_OK || (st = check_bhld(Yk)) != LX_OK) return st;
    if (!same_shape(Q, Yq) || !same_shape(Q, Yk)) return LX_ERR_INVALID;
  }
  if (!al16(wq) || !al16(wk) || !al16(table) || !al16(mq) || !al16(mk)) return LX_ERR_ALIGN;
  if (qc && (!al16(qc) || !al16(kc) || !al16(qs) || !al16(ks))) return LX_ERR_ALIGN;
  lx::ProParams pro{};
  pro.wq = wq;
  pro.wk = wk;
  pro.table = reinterpret_cast<const float2*>(table);
  if (Yq) {
    pro.yq = lx::BhldOut{reinterpret_cast<__nv_bfloat16*>(Yq->data), Yq->sB, Yq->sH, Yq->sL};
    pro.yk = lx::BhldOut{reinterpret_cast<__nv_bfloat16*>(Yk->data), Yk->sB, Yk->sH, Yk->sL};
  }
  pro.eps = eps;
  pro.Hh = (int)rope->Hh;
  pro.W = (int)rope->W;
  pro.dt2 = rope->dt / 2;
  pro.dh2 = rope->dh / 2;
  pro.offh = (int)(rope->T * (rope->dt / 2));
  pro.offw = pro.offh + (int)(rope->Hh * (rope->dh / 2));
  return Q->D == 128 ? launch_qk_pass<128>(Q, K, mq, mk, qc, qs, kc, ks, stream, &pro)
                     : launch_qk_pass<64>(Q, K, mq, mk, qc, qs, kc, ks, stream, &pro);
}

// ---------------------------------------------------------------- K smoothing (variant)
lx_status lx_k_channel_mean_ws_size(const lx_bhld* K, size_t* bytes) {
  lx_status st = check_bhld(K);
  if (st != LX_OK) return st;
  if (!bytes) return LX_ERR_INVALID;
  const int64_t nSpan = (K->L + lx::kVSpan - 1) / lx::kVSpan;
  *bytes = sizeof(double) * (size_t)(K->B * K->H * nSpan * K->D);
  return LX_OK;
}

lx_status lx_k_channel_mean(const lx_bhld* K, void* ws, size_t ws_bytes, float* km, cudaStream_t stream) {
  size_t need = 0;
  lx_status st = lx_k_channel_mean_ws_size(K, &need);
  if (st != LX_OK) return st;
  if (!km) return LX_ERR_INVALID;
  if (!ws || ws_bytes < need) return LX_ERR_WORKSPACE;
  if (!al16(ws) || !al16(km)) return LX_ERR_ALIGN;
  const int64_t BH = K->B * K->H;
  const int nSpan = (int)((K->L + lx::kVSpan - 1) / lx::kVSpan);
  double* part = reinterpret_cast<double*>(ws);
  if (K->D == 128)
    lx::k_mean_partial_kernel<128><<<(unsigned)(BH * nSpan), 128, 0, stream>>>(view(K), part, (int)K->H, (int)K->L, nSpan);
  else
    lx::k_mean_partial_kernel<64><<<(unsigned)(BH * nSpan), 128, 0, stream>>>(view(K), part, (int)K->H, (int)K->L, nSpan);
  if (cudaGetLastError() != cudaSuccess) return LX_ERR_CUDA;
  const long long n = BH * K->D;
  lx::k_mean_final_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(part, km, BH, (int)K->D, nSpan, (int)K->L);
  return launch_status();
}

lx_status lx_quantize_qk_smooth(const lx_bhld* Q, const lx_bhld* K, const float* km, int8_t* qc, float* qs, int8_t* kc,
                                float* ks, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK) return st;
  if (!same_shape(Q, K) || !km || !qc || !qs || !kc || !ks) return LX_ERR_INVALID;
  if (!al16(km) || !al16(qc) || !al16(kc) || !al16(qs) || !al16(ks)) return LX_ERR_ALIGN;
  if (Q->D == 128)
    launch_smooth<128, false>(Q, K, km, nullptr, nullptr, qc, qs, kc, ks, stream);
  else
    launch_smooth<64, false>(Q, K, km, nullptr, nullptr, qc, qs, kc, ks, stream);
  return launch_status();
}

lx_status lx_pool_quantize_qk_smooth(const lx_bhld* Q, const lx_bhld* K, const float* km, float* mq, float* mk,
                                     int8_t* qc, float* qs, int8_t* kc, float* ks, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK) return st;
  if (!same_shape(Q, K) || !km || !mq || !mk || !qc || !qs || !kc || !ks) return LX_ERR_INVALID;
  if (!al16(km) || !al16(mq) || !al16(mk) || !al16(qc) || !al16(kc) || !al16(qs) || !al16(ks)) return LX_ERR_ALIGN;
  if (Q->D == 128)
    launch_smooth<128, true>(Q, K, km, mq, mk, qc, qs, kc, ks, stream);
  else
    launch_smooth<64, true>(Q, K, km, mq, mk, qc, qs, kc, ks, stream);
  return launch_status();
}

lx_status lx_quantize_v(const lx_bhld* V, uint8_t* vc, float* vs, uint32_t* amax_ws, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(V)) != LX_OK) return st;
  if (!vc || !vs || !amax_ws) return LX_ERR_INVALID;
  if (!al16(vc) || !al16(vs) || !al16(amax_ws)) return LX_ERR_ALIGN;
  return V->D == 128 ? launch_quant_v<128>(V, vc, vs, amax_ws, stream)
                     : launch_quant_v<64>(V, vc, vs, amax_ws, stream);
}

// Built-in V absmax scratch of lx_quantize_v_noalloc (one copy per device).
static __device__ __align__(256) uint32_t g_noalloc_amax[LX_NOALLOC_AMAX_MAX];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
// Per device: the context the address was looked up in, and the address.  A
// device reset gives the device a new primary context whose copy of the array
// may sit elsewhere, so a cached address is reused only in the same context.
struct NoallocEntry {
  CUcontext ctx;
  uint32_t* ptr;
};
NoallocEntry g_noalloc[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  return fn;
}

// Device address of g_noalloc_amax on the current device, looked up once per
// (device, context).
lx_status noalloc_scratch(uint32_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return LX_ERR_CUDA;
  if (dev >= kMaxDevices) return LX_ERR_UNSUPPORTED;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (!get_ctx) return LX_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocEntry& e = g_noalloc[dev];
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return LX_ERR_CUDA;
  if (!e.ptr || !ctx || e.ctx != ctx) {
    // the lookup also makes the runtime's context current when none is yet
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_amax) != cudaSuccess || !p) return LX_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return LX_ERR_CUDA;
    e.ctx = ctx;
    e.ptr = static_cast<uint32_t*>(p);
  }
  *out = e.ptr;
  return LX_OK;
}
}  // namespace

lx_status lx_quantize_v_noalloc(const lx_bhld* V, uint8_t* vc, float* vs, cudaStream_t stream) {
  lx_status st = check_bhld(V);
  if (st != LX_OK) return st;
  if (!vc || !vs) return LX_ERR_INVALID;
  if (!al16(vc) || !al16(vs)) return LX_ERR_ALIGN;
  if (V->B * V->H * V->D > (int64_t)LX_NOALLOC_AMAX_MAX) return LX_ERR_WORKSPACE;
  uint32_t* amax = nullptr;
  if ((st = noalloc_scratch(&amax)) != LX_OK) return st;
  return V->D == 128 ? launch_quant_v<128>(V, vc, vs, amax, stream) : launch_quant_v<64>(V, vc, vs, amax, stream);
}

lx_status lx_attn_bf16(const lx_bhld* Q, const lx_bhld* K, const lx_bhld* V, const lx_plan* plan, const lx_bhld* O,
                       cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK || (st = check_bhld(V)) != LX_OK ||
      (st = check_bhld(O)) != LX_OK)
    return st;
  if (!same_shape(Q, K) || !same_shape(Q, V) || !same_shape(Q, O)) return LX_ERR_INVALID;
  if ((st = check_plan(plan, Q)) != LX_OK) return st;
  return Q->D == 128 ? attn_bf16_impl<128>(Q, K, V, plan, O, stream) : attn_bf16_impl<64>(Q, K, V, plan, O, stream);
}

lx_status lx_attn_int8fp8(const int8_t* qc, const float* qs, const int8_t* kc, const float* ks, const uint8_t* vc,
                          const float* vs, const lx_plan* plan, const lx_bhld* O, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(O)) != LX_OK) return st;
  if (!qc || !qs || !kc || !ks || !vc || !vs) return LX_ERR_INVALID;
  if (!al16(qc) || !al16(kc) || !al16(vc) || !al16(qs) || !al16(ks) || !al16(vs)) return LX_ERR_ALIGN;
  if ((st = check_plan(plan, O)) != LX_OK) return st;
  return O->D == 128 ? attn_i8_impl<128>(qc, qs, kc, ks, vc, vs, plan, O, stream)
                     : attn_i8_impl<64>(qc, qs, kc, ks, vc, vs, plan, O, stream);
}

lx_status lx_fwd_workspace_size(const lx_bhld* Q, lx_mode mode, size_t* bytes) {
  if (!Q || !bytes) return LX_ERR_INVALID;
  if (Q->B < 1 || Q->H < 1 || Q->L < 1) return LX_ERR_INVALID;
  if (Q->D != 64 && Q->D != 128) return LX_ERR_UNSUPPORTED;
  if (mode == LX_MODE_BF16) {
    *bytes = 0;
    return LX_OK;
  }
  if (mode != LX_MODE_INT8FP8) return LX_ERR_INVALID;
  *bytes = fwd_layout(Q).total;
  return LX_OK;
}

lx_status lx_sparse_attn_fwd(const lx_bhld* Q, const lx_bhld* K, const lx_bhld* V, const lx_plan* plan, lx_mode mode,
                             const lx_bhld* O, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (mode == LX_MODE_BF16) return lx_attn_bf16(Q, K, V, plan, O, stream);
  if (mode != LX_MODE_INT8FP8) return LX_ERR_INVALID;
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK || (st = check_bhld(V)) != LX_OK ||
      (st = check_bhld(O)) != LX_OK)
    return st;
  if (!same_shape(Q, K) || !same_shape(Q, V) || !same_shape(Q, O)) return LX_ERR_INVALID;
  if ((st = check_plan(plan, Q)) != LX_OK) return st;
  const FwdWs w = fwd_layout(Q);
  if (!ws || ws_bytes < w.total) return LX_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return LX_ERR_ALIGN;
  char* base = reinterpret_cast<char*>(ws);
  int8_t* qc = reinterpret_cast<int8_t*>(base + w.qc);
  int8_t* kc = reinterpret_cast<int8_t*>(base + w.kc);
  uint8_t* vc = reinterpret_cast<uint8_t*>(base + w.vc);
  float* qs = reinterpret_cast<float*>(base + w.qs);
  float* ks = reinterpret_cast<float*>(base + w.ks);
  float* vs = reinterpret_cast<float*>(base + w.vs);
  uint32_t* amax = reinterpret_cast<uint32_t*>(base + w.amax);
  if ((st = lx_quantize_qk(Q, K, qc, qs, kc, ks, stream)) != LX_OK) return st;
  if ((st = lx_quantize_v(V, vc, vs, amax, stream)) != LX_OK) return st;
  return lx_attn_int8fp8(qc, qs, kc, ks, vc, vs, plan, O, stream);
}

lx_status lx_sparse_attn_ws_size(const lx_bhld* Q, double keep, lx_mode mode, size_t* bytes) {
  if (!Q || !bytes) return LX_ERR_INVALID;
  size_t plan_ws = 0, fwd_ws = 0;
  lx_status st = lx_plan_size(Q->B, Q->H, Q->L, Q->D, keep, nullptr, nullptr, nullptr, &plan_ws);
  if (st != LX_OK) return st;
  if ((st = lx_fwd_workspace_size(Q, mode, &fwd_ws)) != LX_OK) return st;
  *bytes = align256(plan_ws) + fwd_ws;
  return LX_OK;
}

lx_status lx_sparse_attn(const lx_bhld* Q, const lx_bhld* K, const lx_bhld* V, double keep, lx_mode mode,
                         lx_plan* plan, const lx_bhld* O, void* ws, size_t ws_bytes, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(Q)) != LX_OK || (st = check_bhld(K)) != LX_OK || (st = check_bhld(V)) != LX_OK ||
      (st = check_bhld(O)) != LX_OK)
    return st;
  if (!same_shape(Q, K) || !same_shape(Q, V) || !same_shape(Q, O) || !plan) return LX_ERR_INVALID;
  if (mode != LX_MODE_BF16 && mode != LX_MODE_INT8FP8) return LX_ERR_INVALID;
  size_t need = 0, plan_ws = 0;
  if ((st = lx_sparse_attn_ws_size(Q, keep, mode, &need)) != LX_OK) return st;
  if ((st = lx_plan_size(Q->B, Q->H, Q->L, Q->D, keep, nullptr, nullptr, nullptr, &plan_ws)) != LX_OK) return st;
  if (!ws || ws_bytes < need) return LX_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return LX_ERR_ALIGN;
  if (n_blocks(Q->L) > kMaxPlannerNB) return LX_ERR_UNSUPPORTED;
  // workspace: [means of Q | means of K | scores (planner) | codes and scales (forward)]
  char* base = reinterpret_cast<char*>(ws);
  const size_t means = align256(sizeof(float) * (size_t)(Q->B * Q->H * n_blocks(Q->L) * Q->D));
  float* mq = reinterpret_cast<float*>(base);
  float* mk = reinterpret_cast<float*>(base + means);
  char* sc = base + 2 * means;
  const size_t sc_bytes = plan_ws - 2 * means;
  if (mode == LX_MODE_BF16) {
    if ((st = lx_pool_means(Q, K, mq, mk, stream)) != LX_OK) return st;
    if ((st = lx_score_topk(mq, mk, Q->B, Q->H, Q->L, Q->D, keep, plan, sc, sc_bytes, stream)) != LX_OK) return st;
    return lx_attn_bf16(Q, K, V, plan, O, stream);
  }
  const FwdWs w = fwd_layout(Q);
  char* fb = base + align256(plan_ws);
  int8_t* qc = reinterpret_cast<int8_t*>(fb + w.qc);
  int8_t* kc = reinterpret_cast<int8_t*>(fb + w.kc);
  uint8_t* vc = reinterpret_cast<uint8_t*>(fb + w.vc);
  float* qs = reinterpret_cast<float*>(fb + w.qs);
  float* ks = reinterpret_cast<float*>(fb + w.ks);
  float* vs = reinterpret_cast<float*>(fb + w.vs);
  uint32_t* amax = reinterpret_cast<uint32_t*>(fb + w.amax);
  // Q and K are read once for the block means and the INT8 codes
  if ((st = lx_pool_quantize_qk(Q, K, mq, mk, qc, qs, kc, ks, stream)) != LX_OK) return st;
  if ((st = lx_score_topk(mq, mk, Q->B, Q->H, Q->L, Q->D, keep, plan, sc, sc_bytes, stream)) != LX_OK) return st;
  if ((st = lx_quantize_v(V, vc, vs, amax, stream)) != LX_OK) return st;
  return lx_attn_int8fp8(qc, qs, kc, ks, vc, vs, plan, O, stream);
}

lx_status lx_last_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return LX_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, lx::g_device_status, sizeof(int)) != cudaSuccess) return LX_ERR_CUDA;
  const int zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(lx::g_device_status, &zero, sizeof(int)) != cudaSuccess) return LX_ERR_CUDA;
  if (v == LX_ERR_TIMEOUT || v == LX_ERR_PLAN) return (lx_status)v;
  return v == 0 ? LX_OK : LX_ERR_CUDA;
}

lx_status lx_debug_wait_timeout(uint64_t limit_ns, cudaStream_t stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return LX_ERR_INVALID;
  lx::wait_timeout_probe_kernel<<<1, 32, 0, stream>>>((unsigned long long)limit_ns);
  return launch_status();
}

// ---------------------------------------------------------------- Light-Ulysses exchange
namespace {
// rows of one destination's segment, its scale offset and its size (16-byte rounded)
void ulysses_segment(int64_t B, int64_t hc, int64_t Lr, int64_t D, int64_t X, long long* rows_r, long long* sc_off,
                     long long* seg) {
  *rows_r = (long long)B * hc * Lr * X;
  *sc_off = (*rows_r * D + 15) / 16 * 16;
  *seg = *sc_off + (*rows_r * 4 + 15) / 16 * 16;
}
}  // namespace

lx_status lx_ulysses_segment_bytes(int64_t B, int64_t hc, int64_t Lr, int64_t D, int64_t tensors, size_t* seg_bytes) {
  if (!seg_bytes || B < 1 || hc < 1 || Lr < 1 || (D != 64 && D != 128) || (tensors != 1 && tensors != 3))
    return LX_ERR_INVALID;
  long long rows_r, sc_off, seg;
  ulysses_segment(B, hc, Lr, D, tensors, &rows_r, &sc_off, &seg);
  *seg_bytes = (size_t)seg;
  return LX_OK;
}

lx_status lx_ulysses_pack_qkv(const lx_bhld* q, const lx_bhld* k, const lx_bhld* v, int64_t N, int64_t h0, int64_t hc,
                              uint8_t* payload, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(q)) != LX_OK || (st = check_bhld(k)) != LX_OK || (st = check_bhld(v)) != LX_OK) return st;
  if (!same_shape(q, k) || !same_shape(q, v) || !payload) return LX_ERR_INVALID;
  if (N < 1 || q->H % N != 0 || h0 < 0 || hc < 1 || h0 + hc > q->H / N) return LX_ERR_INVALID;
  if (!al16(payload)) return LX_ERR_ALIGN;
  lx::UlyssesArgs a{};
  a.x[0] = rw(q);
  a.x[1] = rw(k);
  a.x[2] = rw(v);
  a.payload = payload;
  long long rows_r;
  ulysses_segment(q->B, hc, q->L, q->D, 3, &rows_r, &a.sc_off, &a.seg);
  a.N = (int)N;
  a.B = (int)q->B;
  a.Hr = (int)(q->H / N);
  a.Hc = (int)hc;
  a.h0 = (int)h0;
  a.Lr = (int)q->L;
  a.rows = (long long)N * rows_r;
  return launch_ulysses<lx::kPackQKV>(a, q->D, stream);
}

lx_status lx_ulysses_unpack_qkv(const uint8_t* payload, int64_t N, const lx_bhld* q, const lx_bhld* k,
                                const lx_bhld* v, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(q)) != LX_OK || (st = check_bhld(k)) != LX_OK || (st = check_bhld(v)) != LX_OK) return st;
  if (!same_shape(q, k) || !same_shape(q, v) || !payload) return LX_ERR_INVALID;
  if (N < 1 || q->L % N != 0) return LX_ERR_INVALID;
  if (!al16(payload)) return LX_ERR_ALIGN;
  lx::UlyssesArgs a{};
  a.x[0] = rw(q);
  a.x[1] = rw(k);
  a.x[2] = rw(v);
  a.payload = const_cast<uint8_t*>(payload);
  long long rows_r;
  ulysses_segment(q->B, q->H, q->L / N, q->D, 3, &rows_r, &a.sc_off, &a.seg);
  a.N = (int)N;
  a.B = (int)q->B;
  a.Hr = (int)q->H;
  a.Hc = (int)q->H;
  a.Lr = (int)(q->L / N);
  a.rows = (long long)N * rows_r;
  return launch_ulysses<lx::kUnpackQKV>(a, q->D, stream);
}

lx_status lx_ulysses_pack_o(const lx_bhld* o, int64_t N, uint8_t* payload, cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(o)) != LX_OK) return st;
  if (!payload || N < 1 || o->L % N != 0) return LX_ERR_INVALID;
  if (!al16(payload)) return LX_ERR_ALIGN;
  lx::UlyssesArgs a{};
  a.x[0] = rw(o);
  a.payload = payload;
  long long rows_r;
  ulysses_segment(o->B, o->H, o->L / N, o->D, 1, &rows_r, &a.sc_off, &a.seg);
  a.N = (int)N;
  a.B = (int)o->B;
  a.Hr = (int)o->H;
  a.Hc = (int)o->H;
  a.Lr = (int)(o->L / N);
  a.rows = (long long)N * rows_r;
  return launch_ulysses<lx::kPackO>(a, o->D, stream);
}

lx_status lx_ulysses_unpack_o(const uint8_t* payload, int64_t N, int64_t h0, int64_t hc, const lx_bhld* out,
                              cudaStream_t stream) {
  lx_status st;
  if ((st = check_bhld(out)) != LX_OK) return st;
  if (!payload || N < 1 || out->H % N != 0 || h0 < 0 || hc < 1 || h0 + hc > out->H / N) return LX_ERR_INVALID;
  if (!al16(payload)) return LX_ERR_ALIGN;
  lx::UlyssesArgs a{};
  a.x[0] = rw(out);
  a.payload = const_cast<uint8_t*>(payload);
  long long rows_r;
  ulysses_segment(out->B, hc, out->L, out->D, 1, &rows_r, &a.sc_off, &a.seg);
  a.N = (int)N;
  a.B = (int)out->B;
  a.Hr = (int)(out->H / N);
  a.Hc = (int)hc;
  a.h0 = (int)h0;
  a.Lr = (int)out->L;
  a.rows = (long long)N * rows_r;
  return launch_ulysses<lx::kUnpackO>(a, out->D, stream);
}

// ---------------------------------------------------------------- NVFP4
lx_status lx_nvfp4_sizes(int64_t R, int64_t K, size_t* code_bytes, size_t* sf_bytes) {
  if (R < 1 || K < 64 || K % 64 != 0 || K > ((int64_t)1 << 30)) return LX_ERR_INVALID;
  if (code_bytes) *code_bytes = (size_t)R * (size_t)(K / 2);
  if (sf_bytes) *sf_bytes = (size_t)((R + 127) / 128) * 128 * (size_t)(K / 16);
  return LX_OK;
}

lx_status lx_nvfp4_quantize(const void* x, int64_t R, int64_t K, int64_t ldx, int compute_gscale, float* gscale,
                            uint8_t* codes, uint8_t* sf, cudaStream_t stream) {
  if (!x || !gscale || !codes || !sf) return LX_ERR_INVALID;
  if (R < 1 || K < 64 || K % 64 != 0 || K > ((int64_t)1 << 30) || ldx < K) return LX_ERR_INVALID;
  const int64_t tiles = (R + 127) / 128, ysteps = (K / 64 + lx::kNvQSteps - 1) / lx::kNvQSteps;
  if (tiles > 0x7FFFFFFF || ysteps > 65535) return LX_ERR_UNSUPPORTED;
  if (!al16(x) || ldx % 8 != 0 || !al16(codes) || !al16(sf) || (reinterpret_cast<uintptr_t>(gscale) & 3u))
    return LX_ERR_ALIGN;
  const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  if (compute_gscale) {
    if (cudaMemsetAsync(gscale, 0, sizeof(float), stream) != cudaSuccess) return LX_ERR_CUDA;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return LX_ERR_CUDA;
    const int64_t ctas = R < 8LL * sms ? R : 8LL * sms;
    lx::nvfp4_amax_kernel<<<(unsigned)ctas, 256, 0, stream>>>(xb, R, (int)K, ldx, reinterpret_cast<unsigned*>(gscale));
    lx::nvfp4_gscale_kernel<<<1, 1, 0, stream>>>(gscale);
  }
  lx::nvfp4_quant_kernel<<<dim3((unsigned)tiles, (unsigned)ysteps), 128, 0, stream>>>(xb, R, (int)K, ldx, gscale,
                                                                                       codes, sf);
  return launch_status();
}

lx_status lx_nvfp4_gemm(const uint8_t* xc, const uint8_t* xsf, const float* gx, const uint8_t* wc,
                        const uint8_t* wsf, const float* gw, const float* bias, int64_t M, int64_t N, int64_t K,
                        void* y, int64_t ldy, cudaStream_t stream) {
  if (!xc || !xsf || !gx || !wc || !wsf || !gw || !y) return LX_ERR_INVALID;
  if (M < 1 || N < 128 || N % 128 != 0 || K < 256 || K % 256 != 0 || ldy < N) return LX_ERR_INVALID;
  const int64_t mtiles = (M + lx::kNvBM - 1) / lx::kNvBM, ntiles = (N + lx::kNvBN - 1) / lx::kNvBN;
  // row and column coordinates of the TMA loads and the kernel's sizes are 32-bit
  if (M > ((int64_t)1 << 31) - 256 || N > ((int64_t)1 << 31) - 256 || K > ((int64_t)1 << 30))
    return LX_ERR_UNSUPPORTED;
  if (!al16(xc) || !al16(xsf) || !al16(wc) || !al16(wsf) || !al16(y) || ldy % 8 != 0 ||
      (reinterpret_cast<uintptr_t>(gx) & 3u) || (reinterpret_cast<uintptr_t>(gw) & 3u) ||
      (reinterpret_cast<uintptr_t>(bias) & 3u))
    return LX_ERR_ALIGN;
  CUtensorMap ta, tw;
  if (!make_map_codes(&ta, xc, M, K, lx::kNvBM) || !make_map_codes(&tw, wc, N, K, lx::kNvBN)) return LX_ERR_CUDA;
  if (cudaFuncSetAttribute(lx::nvfp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lx::kNvSmemBytes) !=
      cudaSuccess)
    return LX_ERR_CUDA;
  lx::NvGemmArgs a{};
  a.sfa = xsf;
  a.sfb = wsf;
  a.gx = gx;
  a.gw = gw;
  a.bias = bias;
  a.y = reinterpret_cast<__nv_bfloat16*>(y);
  a.ldy = ldy;
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.limit_ns = kWaitLimitNs;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms < 1)
    return LX_ERR_CUDA;
  const int64_t tiles = mtiles * ntiles;  // persistent: one CTA per SM walks the tiles
  const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
  lx::nvfp4_gemm_kernel<<<grid, lx::kNvThreads, lx::kNvSmemBytes, stream>>>(ta, tw, a);
  return launch_status();
}

}  // extern "C"

