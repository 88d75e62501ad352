// C-ABI entry points of libcosa.so: argument validation, workspace layout and
// kernel launches.  All arithmetic of the method runs in the kernels included
// below; this file only checks sizes and marshals pointers.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kap.cuh"
#include "kap_tc.cuh"
#include "attn_tc.cuh"
#include "attn_dense.cuh"
#include "attn_gqa.cuh"
#include "decode.cuh"

using namespace cosa;

namespace {

constexpr int kVersion = (0 << 16) | (1 << 8) | 0;

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

cosa_status_t check_shape(const cosa_shape_t* s) {
  if (!s) return COSA_ERR_INVALID_ARG;
  if (s->batch <= 0 || s->num_q_heads <= 0 || s->num_kv_heads <= 0 || s->seq_len <= 0 ||
      s->head_dim <= 0 || s->page_size <= 0 || s->q_block <= 0 || s->pages_per_seq <= 0 ||
      s->num_phys_pages <= 0)
    return COSA_ERR_INVALID_ARG;
  if (!(s->softmax_scale > 0.f) || !std::isfinite(s->softmax_scale)) return COSA_ERR_INVALID_ARG;
  if (s->num_q_heads % s->num_kv_heads) return COSA_ERR_INVALID_ARG;
  if (s->seq_len % s->page_size || s->seq_len % s->q_block) return COSA_ERR_INVALID_ARG;
  if (s->pages_per_seq < s->seq_len / s->page_size) return COSA_ERR_INVALID_ARG;
  if (s->head_dim != 64 && s->head_dim != 128) return COSA_ERR_UNSUPPORTED;
  if (s->page_size != 64 && s->page_size != 128) return COSA_ERR_UNSUPPORTED;
  if (s->q_block != 64 && s->q_block != 128) return COSA_ERR_UNSUPPORTED;
  // index arithmetic stays in 32 bits for token/page counts, 64 bits for offsets
  if ((long long)s->seq_len > (1ll << 30)) return COSA_ERR_UNSUPPORTED;
  return COSA_OK;
}

cosa_status_t check_kap(const cosa_shape_t* s, const cosa_kap_params_t* k) {
  if (!k) return COSA_ERR_INVALID_ARG;
  if (!(k->budget >= 0.f && k->budget <= 1.f)) return COSA_ERR_INVALID_ARG;
  if (k->q_sub <= 0 || k->k_sub <= 0 || k->sink_pages < 0) return COSA_ERR_INVALID_ARG;
  if (k->ascending != 0 && k->ascending != 1) return COSA_ERR_INVALID_ARG;
  if (s->q_block % k->q_sub || s->page_size % k->k_sub) return COSA_ERR_INVALID_ARG;
  int R = s->q_block / k->q_sub, T = s->page_size / k->k_sub;
  if (!is_pow2(R) || R > 8 || !is_pow2(T) || T > 8) return COSA_ERR_UNSUPPORTED;
  return COSA_OK;
}

struct KapLayout {
  size_t q_hi, q_lo, k_hi, k_lo, a, row_max, row_arg, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of cosa_kap_select: pooled queries and keys (TF32 hi and lo
// terms), the triangular page-max array, and per representative row its max
// and the first page attaining it.
KapLayout kap_layout(const cosa_shape_t* s, const cosa_kap_params_t* k) {
  KapLayout L;
  const size_t B = s->batch, Hq = s->num_q_heads, Hk = s->num_kv_heads, N = s->seq_len,
               D = s->head_dim;
  const size_t R = s->q_block / k->q_sub, nQB = N / s->q_block, nP = N / s->page_size;
  const size_t T = s->page_size / k->k_sub, GR = (Hq / Hk) * R;
  const size_t qrows = B * Hq * nQB * R, krows = B * Hk * nP * T;
  const size_t tri = (size_t)cum_pages((int)nQB, s->q_block, s->page_size);
  size_t off = 0;
  L.q_hi = off;
  off = align256(off + qrows * D * sizeof(float));
  L.q_lo = off;
  off = align256(off + qrows * D * sizeof(float));
  L.k_hi = off;
  off = align256(off + krows * D * sizeof(float));
  L.k_lo = off;
  off = align256(off + krows * D * sizeof(float));
  L.a = off;
  off = align256(off + B * Hk * GR * tri * sizeof(float));
  L.row_max = off;
  off = align256(off + qrows * sizeof(float));
  L.row_arg = off;
  off = align256(off + qrows * sizeof(int));
  L.total = off;
  return L;
}

int kcap_of(const cosa_shape_t* s, const cosa_kap_params_t* k) {
  int best = 0;
  const int nQB = s->seq_len / s->q_block;
  for (int qb = 0; qb < nQB; ++qb) {
    int v = budget_count(qb, s->q_block, s->page_size, k->sink_pages, k->budget);
    best = v > best ? v : best;
  }
  return best;
}

cosa_status_t last_launch() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    return COSA_ERR_CUDA;
  }
  return COSA_OK;
}

// ---- tensor maps (TMA descriptors) ------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 [z][rows][D] viewed as a 3-D tensor; box = 64 columns x box_rows x 1,
// 128-byte swizzle (the layout the UMMA descriptors expect).
bool make_map(CUtensorMap* m, const void* base, int D, int rows, long long z, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)z};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 [rows][D] as a 2-D tensor; box = 32 columns (128 bytes) x 128 rows, 128-byte swizzle.
bool make_map_f32(CUtensorMap* m, const void* base, int D, long long rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 4};
  cuuint32_t box[2] = {32u, 128u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr unsigned long long kWaitTimeoutNs = 1000000000ull;  // 1 s without progress

template <int D, int T>
cosa_status_t launch_score_tc(const ScoreParams& prm, const CUtensorMap* maps, int grid,
                              cudaStream_t st) {
  using Cfg = ScoreCfg<D>;
  auto kern = kap_score_tc<D, T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Cfg::SMEM_ALLOC) != cudaSuccess)
    return COSA_ERR_CUDA;
  kern<<<grid, 192, Cfg::SMEM_ALLOC, st>>>(maps[0], maps[1], maps[2], maps[3], prm);
  return last_launch();
}

cosa_status_t launch_order(const cosa_shape_t* s, const cosa_kap_params_t* k, bool from_a,
                           const float* scores, const uint8_t* hrm, const KapPageMax& pm,
                           float* scores_out, uint8_t* hrm_out, int32_t* order, int32_t* count,
                           int k_cap, cudaStream_t st, bool group = false) {
  const int N = s->seq_len, P = s->page_size, Bq = s->q_block, nP = N / P, nQB = N / Bq;
  int npow2 = 1;
  while (npow2 < nP) npow2 <<= 1;
  // keys by page, then the kept keys (at least one warp's worth for the register sort)
  const size_t smem = (size_t)(npow2 + (npow2 < 32 ? 32 : npow2)) * 8;
  if (smem > 200 * 1024) return COSA_ERR_UNSUPPORTED;
  if (from_a && (group ? pm.group : 1) * pm.R > ORDER_MAX_ROWS) return COSA_ERR_UNSUPPORTED;
  const int R = s->q_block / k->q_sub;  // a power of two up to 8 (check_kap)
  auto pick = [&](auto g) {
    constexpr bool G = decltype(g)::value;
    return R == 1 ? kap_order_kernel<true, G, 1>
         : R == 2 ? kap_order_kernel<true, G, 2>
         : R == 4 ? kap_order_kernel<true, G, 4> : kap_order_kernel<true, G, 8>;
  };
  auto kern = !from_a ? kap_order_kernel<false, false, 0>
                      : (group ? pick(std::true_type()) : pick(std::false_type()));
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return COSA_ERR_CUDA;
  dim3 grid(nQB, s->batch * (group ? s->num_kv_heads : s->num_q_heads));
  kern<<<grid, ORDER_THREADS, smem, st>>>(scores, hrm, pm, scores_out, hrm_out, order, count,
                                          s->num_q_heads, nQB, nP, Bq, P, k->budget,
                                          k->sink_pages, k->ascending, k_cap);
  return last_launch();
}

// K1: pooling of Q and of the paged K into the workspace
template <int D>
cosa_status_t launch_pool(const cosa_shape_t* s, const cosa_kap_params_t* k, const void* q,
                          const void* k_pool, const int32_t* page_table, const KapLayout& L,
                          uint8_t* ws, cudaStream_t st) {
  const int B = s->batch, Hq = s->num_q_heads, Hk = s->num_kv_heads, N = s->seq_len;
  const int P = s->page_size, Bq = s->q_block, nP = N / P, nQB = N / Bq;
  const int R = Bq / k->q_sub, T = P / k->k_sub, G = Hq / Hk;
  const long long n_qvec = (long long)B * Hq * nQB * R;
  const long long n_kvec = (long long)B * Hk * nP * T;
  const long long blocks = (n_qvec + n_kvec + 7) / 8;
  if (blocks > 0x7fffffffll) return COSA_ERR_UNSUPPORTED;
  kap_pool_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(k_pool),
      page_table, reinterpret_cast<float*>(ws + L.q_hi), reinterpret_cast<float*>(ws + L.q_lo),
      reinterpret_cast<float*>(ws + L.k_hi), reinterpret_cast<float*>(ws + L.k_lo), n_qvec,
      k->q_sub, n_kvec, k->k_sub, Hq, Hk, G, R, nQB, P, nP, s->pages_per_seq,
      s->num_phys_pages, T);
  return last_launch();
}

// K2 + K3 from the pooled vectors in the workspace
template <int D>
cosa_status_t launch_rank(const cosa_shape_t* s, const cosa_kap_params_t* k, int32_t* order,
                          int32_t* count, float* scores, uint8_t* hrm, const KapLayout& L,
                          uint8_t* ws, int k_cap, cudaStream_t st, bool group = false) {
  const int B = s->batch, Hq = s->num_q_heads, Hk = s->num_kv_heads, N = s->seq_len;
  const int P = s->page_size, Bq = s->q_block, nP = N / P, nQB = N / Bq;
  const int R = Bq / k->q_sub, T = P / k->k_sub, G = Hq / Hk;
  float* q_hi = reinterpret_cast<float*>(ws + L.q_hi);
  float* q_lo = reinterpret_cast<float*>(ws + L.q_lo);
  float* k_hi = reinterpret_cast<float*>(ws + L.k_hi);
  float* k_lo = reinterpret_cast<float*>(ws + L.k_lo);
  const long long n_qvec = (long long)B * Hq * nQB * R;
  const long long n_kvec = (long long)B * Hk * nP * T;

  // K2: scores + MaxPool on the tensor cores
  ScoreParams sp;
  std::memset(&sp, 0, sizeof(sp));
  sp.a = reinterpret_cast<float*>(ws + L.a);
  sp.row_max = reinterpret_cast<float*>(ws + L.row_max);
  sp.row_arg = reinterpret_cast<int*>(ws + L.row_arg);
  sp.group = G;
  sp.R = R;
  sp.T = T;
  sp.num_q_blocks = nQB;
  sp.q_block = Bq;
  sp.page_size = P;
  sp.q_sub = k->q_sub;
  sp.k_sub = k->k_sub;
  sp.rows_per_slab = nQB * G * R;
  sp.keys_per_slab = nP * T;
  sp.tiles_per_slab = (sp.rows_per_slab + 127) / 128;
  sp.scale = s->softmax_scale;
  sp.timeout_ns = kWaitTimeoutNs;
  CUtensorMap maps[4];
  if (!make_map_f32(&maps[0], q_hi, D, n_qvec) || !make_map_f32(&maps[1], q_lo, D, n_qvec) ||
      !make_map_f32(&maps[2], k_hi, D, n_kvec) || !make_map_f32(&maps[3], k_lo, D, n_kvec))
    return COSA_ERR_CUDA;
  const long long grid2 = (long long)B * Hk * sp.tiles_per_slab;
  if (grid2 > 0x7fffffffll) return COSA_ERR_UNSUPPORTED;
  cosa_status_t e = COSA_ERR_UNSUPPORTED;
  switch (T) {
    case 1: e = launch_score_tc<D, 1>(sp, maps, (int)grid2, st); break;
    case 2: e = launch_score_tc<D, 2>(sp, maps, (int)grid2, st); break;
    case 4: e = launch_score_tc<D, 4>(sp, maps, (int)grid2, st); break;
    case 8: e = launch_score_tc<D, 8>(sp, maps, (int)grid2, st); break;
  }
  if (e != COSA_OK) return e;

  // K3: MaxNorm + HRM, budgeted selection, ordering
  KapPageMax pm;
  pm.a = sp.a;
  pm.row_max = sp.row_max;
  pm.row_arg = sp.row_arg;
  pm.num_kv_heads = Hk;
  pm.group = G;
  pm.R = R;
  return launch_order(s, k, true, nullptr, nullptr, pm, scores, hrm, order, count, k_cap, st,
                      group);
}

template <int D>
cosa_status_t launch_kap(const cosa_shape_t* s, const cosa_kap_params_t* k, const void* q,
                         const void* k_pool, const int32_t* page_table, int32_t* order,
                         int32_t* count, float* scores, uint8_t* hrm, const KapLayout& L,
                         uint8_t* ws, int k_cap, cudaStream_t st, bool group = false) {
  if (launch_pool<D>(s, k, q, k_pool, page_table, L, ws, st) != COSA_OK) return COSA_ERR_CUDA;
  return launch_rank<D>(s, k, order, count, scores, hrm, L, ws, k_cap, st, group);
}

template <int D, int P>
cosa_status_t launch_tc_t(const cosa_shape_t* s, const TcParams& prm, const void* q,
                          const void* k_pool, const void* v_pool, int grid, cudaStream_t st) {
  using Cfg = TcCfg<D, P>;
  CUtensorMap mq, mk, mv;
  const long long BH = (long long)s->batch * s->num_q_heads;
  const long long PZ = (long long)s->num_phys_pages * s->num_kv_heads;
  if (!make_map(&mq, q, D, s->seq_len, BH, s->q_block) ||
      !make_map(&mk, k_pool, D, P, PZ, P) || !make_map(&mv, v_pool, D, P, PZ, P))
    return COSA_ERR_CUDA;
  auto kern = prm.max_run > 0 ? attn_tc_kernel<D, P, true> : attn_tc_kernel<D, P, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Cfg::SMEM_ALLOC) != cudaSuccess)
    return COSA_ERR_CUDA;
  kern<<<grid, Cfg::NT, Cfg::SMEM_ALLOC, st>>>(mq, mk, mv, prm);
  return last_launch();
}

template <int D, int P>
cosa_status_t launch_dense_t(const cosa_shape_t* s, const TcParams& prm, const void* q,
                             const void* k_pool, const void* v_pool, int grid, cudaStream_t st) {
  using Cfg = DenseCfg<D, P>;
  CUtensorMap mq, mk, mv;
  const long long BH = (long long)s->batch * s->num_q_heads;
  const long long PZ = (long long)s->num_phys_pages * s->num_kv_heads;
  // Q in 64-row boxes: a 128-row tile past the end of the sequence loads its
  // first half only
  if (!make_map(&mq, q, D, s->seq_len, BH, 64) || !make_map(&mk, k_pool, D, P, PZ, P) ||
      !make_map(&mv, v_pool, D, P, PZ, P))
    return COSA_ERR_CUDA;
  auto kern = attn_dense_kernel<D, P>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Cfg::SMEM_ALLOC) != cudaSuccess)
    return COSA_ERR_CUDA;
  kern<<<grid, Cfg::NT, Cfg::SMEM_ALLOC, st>>>(mq, mk, mv, prm);
  return last_launch();
}

template <int D, int P>
cosa_status_t launch_pair_t(const cosa_shape_t* s, const TcParams& prm, const void* q,
                            const void* k_pool, const void* v_pool, int grid, cudaStream_t st) {
  using Cfg = PairCfg<D, P>;
  CUtensorMap mq, mk, mv;
  const long long BH = (long long)s->batch * s->num_q_heads;
  const long long PZ = (long long)s->num_phys_pages * s->num_kv_heads;
  if (!make_map(&mq, q, D, s->seq_len, BH, s->q_block) || !make_map(&mk, k_pool, D, P, PZ, P) ||
      !make_map(&mv, v_pool, D, P, PZ, P))
    return COSA_ERR_CUDA;
  auto kern = attn_pair_kernel<D, P>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Cfg::SMEM_ALLOC) != cudaSuccess)
    return COSA_ERR_CUDA;
  kern<<<grid, Cfg::NT, Cfg::SMEM_ALLOC, st>>>(mq, mk, mv, prm);
  return last_launch();
}

cosa_status_t launch_osk(const cosa_shape_t* s, const TcParams& prm, const void* q,
                         const void* k_pool, const void* v_pool, int grid, cudaStream_t st) {
  const int D = s->head_dim, P = s->page_size;
  if (D == 128 && P == 64) return launch_tc_t<128, 64>(s, prm, q, k_pool, v_pool, grid, st);
  if (D == 128 && P == 128) return launch_tc_t<128, 128>(s, prm, q, k_pool, v_pool, grid, st);
  if (D == 64 && P == 64) return launch_tc_t<64, 64>(s, prm, q, k_pool, v_pool, grid, st);
  if (D == 64 && P == 128) return launch_tc_t<64, 128>(s, prm, q, k_pool, v_pool, grid, st);
  return COSA_ERR_UNSUPPORTED;
}

TcParams make_params(const cosa_shape_t* s, void* out, float* lse, const int32_t* page_table) {
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  p.page_table = page_table;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.num_q_heads = s->num_q_heads;
  p.num_kv_heads = s->num_kv_heads;
  p.group = s->num_q_heads / s->num_kv_heads;
  p.seq_len = s->seq_len;
  p.num_q_blocks = s->seq_len / s->q_block;
  p.pages_per_seq = s->pages_per_seq;
  p.q_block = s->q_block;
  p.scale_log2 = s->softmax_scale * 1.4426950408889634f;
  p.log2_eps = -INFINITY;
  p.max_run = 0;
  p.timeout_ns = kWaitTimeoutNs;
  p.fault_k_group = -1;
  return p;
}

// Workspace of cosa_osk_decode: the listed pages' logits and local maxima, and the
// per-chunk partial sums.
struct DecodeLayout {
  size_t logits, mloc, po, pl, pn, arr, total;
  int n_chunks;
};

DecodeLayout decode_layout(const cosa_shape_t* s, int k_cap) {
  DecodeLayout L;
  const size_t bh = (size_t)s->batch * s->num_q_heads;
  L.n_chunks = (k_cap + DEC_CHUNK - 1) / DEC_CHUNK;
  size_t off = 0;
  L.logits = off;
  off = align256(off + bh * k_cap * s->page_size * sizeof(float));
  L.mloc = off;
  off = align256(off + bh * k_cap * sizeof(float));
  L.po = off;
  off = align256(off + bh * L.n_chunks * s->head_dim * sizeof(float));
  L.pl = off;
  off = align256(off + bh * L.n_chunks * sizeof(float));
  L.pn = off;
  off = align256(off + bh * L.n_chunks * sizeof(int));
  L.arr = off;
  off = align256(off + bh * sizeof(int));
  L.total = off;
  return L;
}

template <int D, int P>
cosa_status_t launch_decode_t(const DecodeParams& prm, int bh, cudaStream_t st) {
  dim3 grid(prm.n_chunks, bh);
  decode_qk_kernel<D, P><<<grid, DEC_THREADS, 0, st>>>(prm);
  if (last_launch() != COSA_OK) return COSA_ERR_CUDA;
  decode_pv_kernel<D, P><<<grid, DEC_THREADS, 0, st>>>(prm);
  return last_launch();
}

// Test hook of cosa_debug_osk_wait_fault: one-shot, per host thread.
struct OskFault {
  bool armed = false;
  int32_t k_group = -1;
  uint64_t wait_limit_ns = 0;
};
thread_local OskFault t_osk_fault;

// ---------------------------------------------------------------------------
// Scratch for cosa_kap_select_noalloc.  Some callers cannot allocate device
// memory at call time (a runtime whose allocator is owned by someone else, a
// pre-planned memory budget, code running where cudaMalloc is not allowed), so
// this entry point uses a fixed array that lives in the library's module: it
// is created on each device when the module loads there and stays until the
// process exits.  Host code only sees a stand-in for it; its device address
// is looked up once per device below.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_kap_noalloc_scratch[COSA_KAP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};  // context the address belongs to

// Unique id of the current CUDA context (0 if it cannot be had): after a device
// reset the library's module loads again in a new context, possibly elsewhere.
unsigned long long current_context_id() {
  using CtxGetCurrent = CUresult (*)(CUcontext*);
  using CtxGetId = CUresult (*)(CUcontext, unsigned long long*);
  static CtxGetCurrent get_cur = nullptr;
  static CtxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrent>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device, looked up with that
// device current on the first call in each context (a device reset starts a new one;
// while no context is current yet, the address is looked up on every call).
cosa_status_t noalloc_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return COSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return COSA_ERR_UNSUPPORTED;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[dev] == nullptr || ctx == 0 || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kap_noalloc_scratch) != cudaSuccess || p == nullptr)
      return COSA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_addr[dev];
  return COSA_OK;
}

// ---------------------------------------------------------------------------
// cosa_attention_host: both stages from host buffers, one KV head at a time.
// Heads are independent in both stages, so KV head c's copies in, its KAP + OSK
// and the copy of its output back run on three streams: the copies of head c + 1
// and the read-back of head c - 1 overlap head c's kernels.  The device copies of
// one head's Q, K, V and output are doubled; the page table, the ordered lists and
// the KAP workspace are single (the kernels use them in stream order).
// ---------------------------------------------------------------------------
size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct HostLayout {
  cosa_shape_t sub;  // one query head with its KV head: H_q = 1, H_kv = 1
  int32_t k_cap;
  size_t q, kv, ord, cnt, pt, kapws;  // bytes: one query head's Q (or O) over the batch, one
                                      // KV head's K (or V) pool column, lists, page table
  size_t off_kv[2][2];                // [set][K, V]
  size_t off_q[3], off_o[3];          // query-head slots
  size_t off_ord, off_cnt, off_kapws, total;  // page table at 0
};
constexpr int kHostQSlots = 3;

cosa_status_t host_layout(const cosa_shape_t* s, const cosa_kap_params_t* kap, HostLayout* L) {
  cosa_status_t e = check_shape(s);
  if (e != COSA_OK) return e;
  if ((e = check_kap(s, kap)) != COSA_OK) return e;
  L->sub = *s;
  L->sub.num_q_heads = 1;
  L->sub.num_kv_heads = 1;
  const cosa_shape_t* u = &L->sub;
  L->k_cap = kcap_of(u, kap);
  const size_t nqb = static_cast<size_t>(u->seq_len / u->q_block);
  const size_t bh = static_cast<size_t>(u->batch);
  L->q = bh * u->seq_len * u->head_dim * 2;
  L->kv = static_cast<size_t>(u->num_phys_pages) * u->page_size * u->head_dim * 2;
  L->ord = bh * nqb * L->k_cap * 4;
  L->cnt = bh * nqb * 4;
  L->pt = static_cast<size_t>(s->batch) * s->pages_per_seq * 4;
  L->kapws = kap_layout(u, kap).total;
  size_t off = al256(L->pt);
  for (int x = 0; x < 2; ++x)
    for (int t = 0; t < 2; ++t) {
      L->off_kv[x][t] = off;
      off += al256(L->kv);
    }
  for (int y = 0; y < kHostQSlots; ++y) {
    L->off_q[y] = off;
    off += al256(L->q);
    L->off_o[y] = off;
    off += al256(L->q);
  }
  L->off_ord = off;
  L->off_cnt = L->off_ord + al256(L->ord);
  L->off_kapws = L->off_cnt + al256(L->cnt);
  L->total = L->off_kapws + al256(L->kapws);
  return COSA_OK;
}

// Streams and events of one cosa_attention_host call, released on scope exit (CUDA
// defers the release of a stream or event until the work queued on it is done).
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, fin_in = nullptr, fin_out = nullptr;
  cudaEvent_t kv_loaded[2] = {}, kv_used[2] = {};
  cudaEvent_t q_loaded[kHostQSlots] = {}, q_used[kHostQSlots] = {}, o_drained[kHostQSlots] = {};
  cudaEvent_t* all(int i) {
    cudaEvent_t* evs[] = {&start, &fin_in, &fin_out, &kv_loaded[0], &kv_loaded[1], &kv_used[0],
                          &kv_used[1], &q_loaded[0], &q_loaded[1], &q_loaded[2], &q_used[0],
                          &q_used[1], &q_used[2], &o_drained[0], &o_drained[1], &o_drained[2]};
    return evs[i];
  }
  static constexpr int kEvents = 16;
  bool create() {
    if (cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking) != cudaSuccess)
      return false;
    for (int i = 0; i < kEvents; ++i)
      if (cudaEventCreateWithFlags(all(i), cudaEventDisableTiming) != cudaSuccess) return false;
    return true;
  }
  ~HostPipe() {
    for (int i = 0; i < kEvents; ++i)
      if (*all(i)) cudaEventDestroy(*all(i));
    if (in) cudaStreamDestroy(in);
    if (out) cudaStreamDestroy(out);
  }
};
static_assert(kHostQSlots == 3, "the event list above names three slots");

}  // namespace

extern "C" {

const char* cosa_status_string(cosa_status_t st) {
  switch (st) {
    case COSA_OK: return "ok";
    case COSA_ERR_INVALID_ARG: return "invalid argument";
    case COSA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case COSA_ERR_CUDA: return "CUDA error";
    case COSA_ERR_TIMEOUT: return "kernel wait timed out";
    case COSA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int32_t cosa_version(void) { return kVersion; }

cosa_status_t cosa_kap_kcap(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                            int32_t* k_cap) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (!k_cap) return COSA_ERR_INVALID_ARG;
  *k_cap = kcap_of(shape, kap);
  return COSA_OK;
}

cosa_status_t cosa_kap_workspace_size(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                      size_t* bytes) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (!bytes) return COSA_ERR_INVALID_ARG;
  *bytes = kap_layout(shape, kap).total;
  return COSA_OK;
}

cosa_status_t cosa_kap_select(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                              const void* q, const void* k_pool, const int32_t* page_table,
                              int32_t* order, int32_t* count, float* scores, uint8_t* hrm,
                              void* workspace, size_t workspace_bytes, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (!q || !k_pool || !page_table || !order || !count) return COSA_ERR_INVALID_ARG;
  KapLayout L = kap_layout(shape, kap);
  if (!workspace || workspace_bytes < L.total) return COSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return COSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16)
    return COSA_ERR_INVALID_ARG;
  const int k_cap = kcap_of(shape, kap);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  if (shape->head_dim == 128)
    return launch_kap<128>(shape, kap, q, k_pool, page_table, order, count, scores, hrm, L, ws,
                           k_cap, st);
  return launch_kap<64>(shape, kap, q, k_pool, page_table, order, count, scores, hrm, L, ws, k_cap,
                        st);
}

cosa_status_t cosa_kap_pool(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                            const void* q, const void* k_pool, const int32_t* page_table,
                            void* workspace, size_t workspace_bytes, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (!q || !k_pool || !page_table) return COSA_ERR_INVALID_ARG;
  KapLayout L = kap_layout(shape, kap);
  if (!workspace || workspace_bytes < L.total) return COSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return COSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16)
    return COSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  if (shape->head_dim == 128) return launch_pool<128>(shape, kap, q, k_pool, page_table, L, ws, st);
  return launch_pool<64>(shape, kap, q, k_pool, page_table, L, ws, st);
}

cosa_status_t cosa_kap_rank(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                            int32_t* order, int32_t* count, float* scores, uint8_t* hrm,
                            void* workspace, size_t workspace_bytes, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (!order || !count) return COSA_ERR_INVALID_ARG;
  KapLayout L = kap_layout(shape, kap);
  if (!workspace || workspace_bytes < L.total) return COSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return COSA_ERR_WORKSPACE;
  const int k_cap = kcap_of(shape, kap);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  if (shape->head_dim == 128)
    return launch_rank<128>(shape, kap, order, count, scores, hrm, L, ws, k_cap, st);
  return launch_rank<64>(shape, kap, order, count, scores, hrm, L, ws, k_cap, st);
}

cosa_status_t cosa_prefill_write(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                 const void* q_tok, const void* k_tok, const void* v_tok,
                                 const int32_t* page_table, void* q, void* k_pool, void* v_pool,
                                 void* workspace, size_t workspace_bytes, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (!q_tok || !k_tok || !v_tok || !page_table || !q || !k_pool || !v_pool)
    return COSA_ERR_INVALID_ARG;
  const void* bufs[] = {q_tok, k_tok, v_tok, q, k_pool, v_pool};
  for (const void* b : bufs)
    if (reinterpret_cast<uintptr_t>(b) % 16) return COSA_ERR_INVALID_ARG;
  KapLayout L = kap_layout(shape, kap);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (ws && (workspace_bytes < L.total || reinterpret_cast<uintptr_t>(ws) % 256))
    return COSA_ERR_WORKSPACE;
  const int B = shape->batch, Hq = shape->num_q_heads, Hk = shape->num_kv_heads, N = shape->seq_len;
  const int P = shape->page_size, Bq = shape->q_block, nP = N / P, nQB = N / Bq;
  const int R = Bq / kap->q_sub, T = P / kap->k_sub, G = Hq / Hk;
  const long long n_qvec = (long long)B * Hq * nQB * R;
  const long long n_kvec = (long long)B * Hk * nP * T;
  const long long blocks = (n_qvec + n_kvec + 7) / 8;
  if (blocks > 0x7fffffffll) return COSA_ERR_UNSUPPORTED;
  float* f[4] = {nullptr, nullptr, nullptr, nullptr};
  if (ws) {
    f[0] = reinterpret_cast<float*>(ws + L.q_hi);
    f[1] = reinterpret_cast<float*>(ws + L.q_lo);
    f[2] = reinterpret_cast<float*>(ws + L.k_hi);
    f[3] = reinterpret_cast<float*>(ws + L.k_lo);
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  using bf = __nv_bfloat16;
  auto args = [&](auto kern) {
    kern<<<(unsigned)blocks, 256, 0, st>>>(
        static_cast<const bf*>(q_tok), static_cast<const bf*>(k_tok), static_cast<const bf*>(v_tok),
        page_table, static_cast<bf*>(q), static_cast<bf*>(k_pool), static_cast<bf*>(v_pool), f[0],
        f[1], f[2], f[3], n_qvec, kap->q_sub, n_kvec, kap->k_sub, Hq, Hk, G, R, nQB, P, nP,
        shape->pages_per_seq, shape->num_phys_pages, T, N);
  };
  if (shape->head_dim == 128) args(prefill_write_kernel<128>);
  else args(prefill_write_kernel<64>);
  return last_launch();
}

cosa_status_t cosa_kap_preskip(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                               float eps, float margin, int32_t* order, int32_t* count,
                               uint8_t* skip_log, const void* workspace, size_t workspace_bytes,
                               cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (!(eps >= 0.f) || !(margin >= 0.f) || !std::isfinite(margin)) return COSA_ERR_INVALID_ARG;
  if (!order || !count) return COSA_ERR_INVALID_ARG;
  KapLayout L = kap_layout(shape, kap);
  if (!workspace || workspace_bytes < L.total) return COSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return COSA_ERR_WORKSPACE;
  const int k_cap = kcap_of(shape, kap);
  if (k_cap > PRESKIP_THREADS * 32) return COSA_ERR_UNSUPPORTED;  // 32 positions per thread
  const int nQB = shape->seq_len / shape->q_block;
  const long long rows = (long long)shape->batch * shape->num_q_heads;
  if (rows > 65535) return COSA_ERR_UNSUPPORTED;
  const uint8_t* ws = reinterpret_cast<const uint8_t*>(workspace);
  KapPageMax pm;
  std::memset(&pm, 0, sizeof(pm));
  pm.a = reinterpret_cast<const float*>(ws + L.a);
  pm.num_kv_heads = shape->num_kv_heads;
  pm.group = shape->num_q_heads / shape->num_kv_heads;
  pm.R = shape->q_block / kap->q_sub;
  const float log_eps = eps > 0.f ? logf(eps) : -INFINITY;
  dim3 grid(nQB, (unsigned)rows);
  kap_preskip_kernel<<<grid, PRESKIP_THREADS, (size_t)k_cap * sizeof(int),
                       reinterpret_cast<cudaStream_t>(stream)>>>(
      pm, order, count, skip_log, shape->num_q_heads, nQB, shape->q_block, shape->page_size,
      k_cap, log_eps, margin);
  return last_launch();
}

cosa_status_t cosa_kap_select_group(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                    const void* q, const void* k_pool, const int32_t* page_table,
                                    int32_t* order, int32_t* count, float* scores, uint8_t* hrm,
                                    void* workspace, size_t workspace_bytes, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (kap->ascending) return COSA_ERR_UNSUPPORTED;
  if (!q || !k_pool || !page_table || !order || !count) return COSA_ERR_INVALID_ARG;
  KapLayout L = kap_layout(shape, kap);
  if (!workspace || workspace_bytes < L.total) return COSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return COSA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16)
    return COSA_ERR_INVALID_ARG;
  const int k_cap = kcap_of(shape, kap);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  if (shape->head_dim == 128)
    return launch_kap<128>(shape, kap, q, k_pool, page_table, order, count, scores, hrm, L, ws,
                           k_cap, st, true);
  return launch_kap<64>(shape, kap, q, k_pool, page_table, order, count, scores, hrm, L, ws, k_cap,
                        st, true);
}

cosa_status_t cosa_kap_select_noalloc(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                      const void* q, const void* k_pool,
                                      const int32_t* page_table, int32_t* order, int32_t* count,
                                      float* scores, uint8_t* hrm, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (!q || !k_pool || !page_table || !order || !count) return COSA_ERR_INVALID_ARG;
  KapLayout L = kap_layout(shape, kap);
  if (L.total > (size_t)COSA_KAP_NOALLOC_SCRATCH_BYTES) return COSA_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16)
    return COSA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if ((e = noalloc_scratch_address(&scratch)) != COSA_OK) return e;
  const int k_cap = kcap_of(shape, kap);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(scratch);
  if (shape->head_dim == 128)
    return launch_kap<128>(shape, kap, q, k_pool, page_table, order, count, scores, hrm, L, ws,
                           k_cap, st);
  return launch_kap<64>(shape, kap, q, k_pool, page_table, order, count, scores, hrm, L, ws, k_cap,
                        st);
}

cosa_status_t cosa_kap_order(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                             const float* scores, const uint8_t* hrm, int32_t* order,
                             int32_t* count, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if ((e = check_kap(shape, kap)) != COSA_OK) return e;
  if (!scores || !hrm || !order || !count) return COSA_ERR_INVALID_ARG;
  KapPageMax pm;
  std::memset(&pm, 0, sizeof(pm));
  return launch_order(shape, kap, false, scores, hrm, pm, nullptr, nullptr, order, count,
                      kcap_of(shape, kap), reinterpret_cast<cudaStream_t>(stream));
}

cosa_status_t cosa_osk_attention(const cosa_shape_t* shape, const cosa_osk_params_t* osk,
                                 const void* q, const void* k_pool, const void* v_pool,
                                 const int32_t* page_table, const int32_t* order,
                                 const int32_t* count, int32_t k_cap, void* out, float* lse,
                                 int32_t* computed, uint8_t* skip_log, cosa_stream_t stream) {
  const OskFault fault = t_osk_fault;  // the test hook is consumed by this call, whatever it returns
  t_osk_fault = OskFault();
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if (!osk || !(osk->eps >= 0.f) || osk->max_run < 0) return COSA_ERR_INVALID_ARG;
  if (!q || !k_pool || !v_pool || !page_table || !order || !count || !out)
    return COSA_ERR_INVALID_ARG;
  if (k_cap <= 0 || k_cap > shape->seq_len / shape->page_size) return COSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16 ||
      reinterpret_cast<uintptr_t>(v_pool) % 16 || reinterpret_cast<uintptr_t>(out) % 16)
    return COSA_ERR_INVALID_ARG;
  TcParams p = make_params(shape, out, lse, page_table);
  p.order = order;
  p.count = count;
  p.computed = computed;
  p.skip_log = skip_log;
  p.k_cap = k_cap;
  p.log2_eps = osk->eps > 0.f ? log2f(osk->eps) : -INFINITY;
  p.max_run = osk->max_run;
  const long long grid = (long long)shape->batch * shape->num_q_heads * (shape->seq_len / shape->q_block);
  if (grid > 0x7fffffffll) return COSA_ERR_UNSUPPORTED;
  if (fault.armed) {
    if (osk->max_run != 0) return COSA_ERR_INVALID_ARG;
    p.fault_k_group = fault.k_group;
    if (fault.wait_limit_ns) p.timeout_ns = fault.wait_limit_ns;
  }
  return launch_osk(shape, p, q, k_pool, v_pool, (int)grid, reinterpret_cast<cudaStream_t>(stream));
}

cosa_status_t cosa_osk_attention_group(const cosa_shape_t* shape, const cosa_osk_params_t* osk,
                                       const void* q, const void* k_pool, const void* v_pool,
                                       const int32_t* page_table, const int32_t* order,
                                       const int32_t* count, int32_t k_cap, void* out, float* lse,
                                       int32_t* computed, uint8_t* skip_log, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if (!osk || !(osk->eps >= 0.f) || osk->max_run < 0) return COSA_ERR_INVALID_ARG;
  if (osk->max_run != 0) return COSA_ERR_UNSUPPORTED;  // the pair kernel has no early break
  if (!q || !k_pool || !v_pool || !page_table || !order || !count || !out)
    return COSA_ERR_INVALID_ARG;
  if (k_cap <= 0 || k_cap > shape->seq_len / shape->page_size) return COSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16 ||
      reinterpret_cast<uintptr_t>(v_pool) % 16 || reinterpret_cast<uintptr_t>(out) % 16)
    return COSA_ERR_INVALID_ARG;
  TcParams p = make_params(shape, out, lse, page_table);
  p.order = order;
  p.count = count;
  p.computed = computed;
  p.skip_log = skip_log;
  p.k_cap = k_cap;
  p.log2_eps = osk->eps > 0.f ? log2f(osk->eps) : -INFINITY;
  const int G = shape->num_q_heads / shape->num_kv_heads;
  const long long grid = (long long)shape->batch * shape->num_kv_heads *
                         (shape->seq_len / shape->q_block) * ((G + 1) / 2);
  if (grid > 0x7fffffffll) return COSA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int D = shape->head_dim, P = shape->page_size;
  if (D == 128 && P == 64) return launch_pair_t<128, 64>(shape, p, q, k_pool, v_pool, (int)grid, st);
  if (D == 128 && P == 128) return launch_pair_t<128, 128>(shape, p, q, k_pool, v_pool, (int)grid, st);
  if (D == 64 && P == 64) return launch_pair_t<64, 64>(shape, p, q, k_pool, v_pool, (int)grid, st);
  if (D == 64 && P == 128) return launch_pair_t<64, 128>(shape, p, q, k_pool, v_pool, (int)grid, st);
  return COSA_ERR_UNSUPPORTED;
}

cosa_status_t cosa_dense_attention(const cosa_shape_t* shape, const void* q, const void* k_pool,
                                   const void* v_pool, const int32_t* page_table, void* out,
                                   float* lse, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if (!q || !k_pool || !v_pool || !page_table || !out) return COSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16 ||
      reinterpret_cast<uintptr_t>(v_pool) % 16 || reinterpret_cast<uintptr_t>(out) % 16)
    return COSA_ERR_INVALID_ARG;
  TcParams p = make_params(shape, out, lse, page_table);
  // one CTA per pair of 128-row query tiles (the q-block size plays no part)
  const long long grid =
      (long long)shape->batch * shape->num_q_heads * ((shape->seq_len + 255) / 256);
  if (grid > 0x7fffffffll) return COSA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int D = shape->head_dim, P = shape->page_size;
  if (D == 128 && P == 64) return launch_dense_t<128, 64>(shape, p, q, k_pool, v_pool, (int)grid, st);
  if (D == 128 && P == 128) return launch_dense_t<128, 128>(shape, p, q, k_pool, v_pool, (int)grid, st);
  if (D == 64 && P == 64) return launch_dense_t<64, 64>(shape, p, q, k_pool, v_pool, (int)grid, st);
  if (D == 64 && P == 128) return launch_dense_t<64, 128>(shape, p, q, k_pool, v_pool, (int)grid, st);
  return COSA_ERR_UNSUPPORTED;
}

cosa_status_t cosa_osk_decode_workspace_size(const cosa_shape_t* shape, int32_t k_cap,
                                             size_t* bytes) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if (!bytes || k_cap <= 0 || k_cap > shape->seq_len / shape->page_size) return COSA_ERR_INVALID_ARG;
  *bytes = decode_layout(shape, k_cap).total;
  return COSA_OK;
}

cosa_status_t cosa_osk_decode(const cosa_shape_t* shape, const cosa_osk_params_t* osk,
                              const void* q, const void* k_pool, const void* v_pool,
                              const int32_t* page_table, const int32_t* positions,
                              const int32_t* order, const int32_t* count, int32_t k_cap, void* out,
                              float* lse, int32_t* computed, uint8_t* skip_log, void* workspace,
                              size_t workspace_bytes, cosa_stream_t stream) {
  cosa_status_t e = check_shape(shape);
  if (e != COSA_OK) return e;
  if (!osk || !(osk->eps >= 0.f && osk->eps <= 1.f) || osk->max_run < 0) return COSA_ERR_INVALID_ARG;
  if (osk->max_run != 0) return COSA_ERR_UNSUPPORTED;
  if (!q || !k_pool || !v_pool || !page_table || !positions || !order || !count || !out)
    return COSA_ERR_INVALID_ARG;
  if (k_cap <= 0 || k_cap > shape->seq_len / shape->page_size) return COSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16 ||
      reinterpret_cast<uintptr_t>(v_pool) % 16)
    return COSA_ERR_INVALID_ARG;
  const DecodeLayout L = decode_layout(shape, k_cap);
  if (!workspace || workspace_bytes < L.total || reinterpret_cast<uintptr_t>(workspace) % 256)
    return COSA_ERR_WORKSPACE;
  const long long bh = (long long)shape->batch * shape->num_q_heads;
  if (bh > 65535) return COSA_ERR_UNSUPPORTED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.q = reinterpret_cast<const __nv_bfloat16*>(q);
  prm.k_pool = reinterpret_cast<const __nv_bfloat16*>(k_pool);
  prm.v_pool = reinterpret_cast<const __nv_bfloat16*>(v_pool);
  prm.page_table = page_table;
  prm.positions = positions;
  prm.order = order;
  prm.count = count;
  prm.out = reinterpret_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.computed = computed;
  prm.skip_log = skip_log;
  prm.logits = reinterpret_cast<float*>(ws + L.logits);
  prm.mloc = reinterpret_cast<float*>(ws + L.mloc);
  prm.part_o = reinterpret_cast<float*>(ws + L.po);
  prm.part_l = reinterpret_cast<float*>(ws + L.pl);
  prm.part_n = reinterpret_cast<int*>(ws + L.pn);
  prm.arrived = reinterpret_cast<int*>(ws + L.arr);
  prm.num_q_heads = shape->num_q_heads;
  prm.num_kv_heads = shape->num_kv_heads;
  prm.group = shape->num_q_heads / shape->num_kv_heads;
  prm.seq_len = shape->seq_len;
  prm.pages_per_seq = shape->pages_per_seq;
  prm.num_phys_pages = shape->num_phys_pages;
  prm.k_cap = k_cap;
  prm.n_chunks = L.n_chunks;
  prm.scale_log2 = shape->softmax_scale * 1.4426950408889634f;
  prm.log2_eps = osk->eps > 0.f ? log2f(osk->eps) : -INFINITY;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int D = shape->head_dim, P = shape->page_size;
  if (D == 128 && P == 64) return launch_decode_t<128, 64>(prm, (int)bh, st);
  if (D == 128 && P == 128) return launch_decode_t<128, 128>(prm, (int)bh, st);
  if (D == 64 && P == 64) return launch_decode_t<64, 64>(prm, (int)bh, st);
  if (D == 64 && P == 128) return launch_decode_t<64, 128>(prm, (int)bh, st);
  return COSA_ERR_UNSUPPORTED;
}

cosa_status_t cosa_debug_osk_wait_fault(int32_t withhold_k_group, uint64_t wait_limit_ns) {
  if (withhold_k_group < -1) return COSA_ERR_INVALID_ARG;
  t_osk_fault.armed = true;
  t_osk_fault.k_group = withhold_k_group;
  t_osk_fault.wait_limit_ns = wait_limit_ns;
  return COSA_OK;
}

cosa_status_t cosa_get_status(cosa_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return COSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return COSA_ERR_CUDA;
  if (v != 0) {
    int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return COSA_ERR_CUDA;
  }
  return static_cast<cosa_status_t>(v);
}

cosa_status_t cosa_attention_host_workspace_size(const cosa_shape_t* shape,
                                                 const cosa_kap_params_t* kap, size_t* bytes) {
  if (!bytes) return COSA_ERR_INVALID_ARG;
  HostLayout L;
  const cosa_status_t e = host_layout(shape, kap, &L);
  if (e != COSA_OK) return e;
  *bytes = L.total;
  return COSA_OK;
}

cosa_status_t cosa_attention_host(const cosa_shape_t* shape, const cosa_kap_params_t* kap,
                                  const cosa_osk_params_t* osk, const void* q_host,
                                  const void* k_pool_host, const void* v_pool_host,
                                  const int32_t* page_table_host, void* out_host, void* workspace,
                                  size_t workspace_bytes, cosa_stream_t stream) {
  HostLayout L;
  cosa_status_t e = host_layout(shape, kap, &L);
  if (e != COSA_OK) return e;
  if (!osk || !(osk->eps >= 0.f) || osk->max_run < 0) return COSA_ERR_INVALID_ARG;
  if (!q_host || !k_pool_host || !v_pool_host || !page_table_host || !out_host)
    return COSA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < L.total || reinterpret_cast<uintptr_t>(workspace) % 256)
    return COSA_ERR_WORKSPACE;
  // the page table is on the host here, so its entries are checked before anything is queued
  for (int b = 0; b < shape->batch; ++b)
    for (int p = 0; p < shape->seq_len / shape->page_size; ++p) {
      const int32_t v = page_table_host[static_cast<size_t>(b) * shape->pages_per_seq + p];
      if (v < 0 || v >= shape->num_phys_pages) return COSA_ERR_INVALID_ARG;
    }
  const int B = shape->batch, Hq = shape->num_q_heads, Hkv = shape->num_kv_heads, G = Hq / Hkv;
  const size_t head_bytes = static_cast<size_t>(shape->seq_len) * shape->head_dim * 2;  // one (b, h)
  const size_t page_bytes = static_cast<size_t>(shape->page_size) * shape->head_dim * 2;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* pt_d = reinterpret_cast<int32_t*>(ws);
  int32_t* ord_d = reinterpret_cast<int32_t*>(ws + L.off_ord);
  int32_t* cnt_d = reinterpret_cast<int32_t*>(ws + L.off_cnt);
  void* kapws_d = ws + L.off_kapws;
  const uint8_t* qh = static_cast<const uint8_t*>(q_host);
  const uint8_t* kh = static_cast<const uint8_t*>(k_pool_host);
  const uint8_t* vh = static_cast<const uint8_t*>(v_pool_host);
  uint8_t* oh = static_cast<uint8_t*>(out_host);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  HostPipe pp;
  if (!pp.create()) return COSA_ERR_CUDA;
  // the workspace may still be in use by earlier work on the caller's stream
  bool ok = cudaEventRecord(pp.start, st) == cudaSuccess &&
            cudaStreamWaitEvent(pp.in, pp.start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(pp.out, pp.start, 0) == cudaSuccess &&
            cudaMemcpyAsync(pt_d, page_table_host, L.pt, cudaMemcpyHostToDevice, pp.in) ==
                cudaSuccess;
  e = ok ? COSA_OK : COSA_ERR_CUDA;
  // One query head at a time (unit u = c * G + g: KV head c, its query head g), so
  // the last unit's kernels and read-back, which no copy-in overlaps, are short.
  // KV head c's pool columns go into set c % 2, reloaded once the kernels of its
  // last query head are done; query head u's Q and O use slot u % 3, Q reloaded once
  // the unit's kernels are done and O rewritten once its read-back is done.
  for (int c = 0; e == COSA_OK && c < Hkv; ++c) {
    const int x = c & 1;
    uint8_t* k_d = ws + L.off_kv[x][0];
    uint8_t* v_d = ws + L.off_kv[x][1];
    // KV head c's column of the page pools (one page-sized row per physical page)
    ok = (c < 2 || cudaStreamWaitEvent(pp.in, pp.kv_used[x], 0) == cudaSuccess) &&
         cudaMemcpy2DAsync(k_d, page_bytes, kh + c * page_bytes, Hkv * page_bytes, page_bytes,
                           shape->num_phys_pages, cudaMemcpyHostToDevice, pp.in) == cudaSuccess &&
         cudaMemcpy2DAsync(v_d, page_bytes, vh + c * page_bytes, Hkv * page_bytes, page_bytes,
                           shape->num_phys_pages, cudaMemcpyHostToDevice, pp.in) == cudaSuccess &&
         cudaEventRecord(pp.kv_loaded[x], pp.in) == cudaSuccess &&
         cudaStreamWaitEvent(st, pp.kv_loaded[x], 0) == cudaSuccess;
    if (!ok) { e = COSA_ERR_CUDA; break; }
    for (int g = 0; g < G; ++g) {
      const int unit = c * G + g, y = unit % kHostQSlots;
      const int h = c * G + g;
      uint8_t* q_d = ws + L.off_q[y];
      uint8_t* o_d = ws + L.off_o[y];
      // query head h of every sequence in
      ok = unit < kHostQSlots || cudaStreamWaitEvent(pp.in, pp.q_used[y], 0) == cudaSuccess;
      for (int b = 0; ok && b < B; ++b)
        ok = cudaMemcpyAsync(q_d + static_cast<size_t>(b) * head_bytes,
                             qh + (static_cast<size_t>(b) * Hq + h) * head_bytes, head_bytes,
                             cudaMemcpyHostToDevice, pp.in) == cudaSuccess;
      ok = ok && cudaEventRecord(pp.q_loaded[y], pp.in) == cudaSuccess &&
           cudaStreamWaitEvent(st, pp.q_loaded[y], 0) == cudaSuccess &&
           (unit < kHostQSlots || cudaStreamWaitEvent(st, pp.o_drained[y], 0) == cudaSuccess);
      if (!ok) { e = COSA_ERR_CUDA; break; }
      e = cosa_kap_select(&L.sub, kap, q_d, k_d, pt_d, ord_d, cnt_d, nullptr, nullptr, kapws_d,
                          L.kapws, stream);
      if (e != COSA_OK) break;
      e = cosa_osk_attention(&L.sub, osk, q_d, k_d, v_d, pt_d, ord_d, cnt_d, L.k_cap, o_d,
                             nullptr, nullptr, nullptr, stream);
      if (e != COSA_OK) break;
      ok = cudaEventRecord(pp.q_used[y], st) == cudaSuccess &&
           (g < G - 1 || cudaEventRecord(pp.kv_used[x], st) == cudaSuccess) &&
           cudaStreamWaitEvent(pp.out, pp.q_used[y], 0) == cudaSuccess;
      // its output back to its place in out_host
      for (int b = 0; ok && b < B; ++b)
        ok = cudaMemcpyAsync(oh + (static_cast<size_t>(b) * Hq + h) * head_bytes,
                             o_d + static_cast<size_t>(b) * head_bytes, head_bytes,
                             cudaMemcpyDeviceToHost, pp.out) == cudaSuccess;
      ok = ok && cudaEventRecord(pp.o_drained[y], pp.out) == cudaSuccess;
      if (!ok) { e = COSA_ERR_CUDA; break; }
    }
  }
  // the caller's stream holds until everything queued above (copies included) is done
  const bool joined = cudaEventRecord(pp.fin_in, pp.in) == cudaSuccess &&
                      cudaEventRecord(pp.fin_out, pp.out) == cudaSuccess &&
                      cudaStreamWaitEvent(st, pp.fin_in, 0) == cudaSuccess &&
                      cudaStreamWaitEvent(st, pp.fin_out, 0) == cudaSuccess;
  if (e == COSA_OK && !joined) e = COSA_ERR_CUDA;
  return e;
}

}  // extern "C"
