// Stage 1 of CoSA, the Kernel-Aware Proxy (gist.science/pt, "CoSA" technical
// summary, §2.2 "Estágio 1: Kernel-Aware Proxy (KAP)").
//
//   kap_pool_kernel   query / key downsampling ("Ranking de Blocos"): mean of
//                     q_sub consecutive query rows and of k_sub consecutive keys
//                     of each logical page (read through the page table).
//                     HBM-bound: one warp per pooled vector, 16-byte loads.
//                     Each mean is written as two TF32 terms hi + lo (hi the
//                     TF32 rounding of the mean, lo the TF32 rounding of the
//                     rest) for the tensor-core scoring in kap_tc.cuh.
//   kap_score_tc      (kap_tc.cuh) approximate scores and MaxPool over each
//                     page's sub-keys on the tensor cores; per representative
//                     row the page maxima a[r][p], the row max and the first
//                     page attaining it.
//   kap_order_kernel  MaxNorm + HRM flags ("Geração de Flag HRM") from those,
//                     budgeted selection and the computation-order mask
//                     ("Ordenação por Grupo de Flags"): packed 64-bit rank
//                     keys, block bitonic sort, forced pages kept,
//                     scan-compaction.  The same kernel also orders caller-given
//                     scores (cosa_kap_order).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace cosa {

// Pages of the q-blocks before qb: sum_{q < qb} n_b(q), for Bq a multiple of P
// or P a multiple of Bq (offsets of the triangular page-max array).
__host__ __device__ __forceinline__ long long cum_pages(int qb, int q_block, int page_size) {
  if (q_block % page_size == 0) {
    const long long c = q_block / page_size;
    return c * qb * (qb + 1) / 2;
  }
  const long long m = page_size / q_block;  // n_b(q) = ceil((q + 1) / m)
  const long long k = qb / m, rem = qb % m;
  return m * k * (k + 1) / 2 + rem * (k + 1);
}

// TF32 rounding (to nearest, ties away) of an fp32 value, kept in an fp32 container.
__device__ __forceinline__ float to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// ---------------------------------------------------------------------------
// K1: pooling.  Work item w < n_qvec: pooled query vector w of the flattened
// [B][H_q][nQB][R] index, written to row ((b H_kv + h_kv) nQB + qb) G R + g R + r
// of q_hi / q_lo (h = h_kv G + g: the representatives of one KV head group and
// q-block are adjacent); else pooled key vector (w - n_qvec) of the
// [B][H_kv][nP][T] index, written to that row of k_hi / k_lo.  Rows are D fp32.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) kap_pool_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_pool,
    const int32_t* __restrict__ page_table, float* __restrict__ q_hi, float* __restrict__ q_lo,
    float* __restrict__ k_hi, float* __restrict__ k_lo, long long n_qvec, int q_sub,
    long long n_kvec, int k_sub, int num_q_heads, int num_kv_heads, int group, int R,
    int num_q_blocks, int page_size, int num_pages, int pages_per_seq, int num_phys_pages,
    int T) {
  constexpr int LPR = D / 8;     // lanes per row: each lane loads 8 bf16 (16 B)
  constexpr int RPI = 32 / LPR;  // rows covered per warp-wide load
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const __nv_bfloat16* src;
  long long drow;
  float *dhi, *dlo;
  int rows, n_read;
  if (w < n_qvec) {
    src = q + w * (long long)q_sub * D;
    const int r = (int)(w % R);
    long long t1 = w / R;
    const int qb = (int)(t1 % num_q_blocks);
    const long long bhq = t1 / num_q_blocks;
    const int h = (int)(bhq % num_q_heads);
    const int b = (int)(bhq / num_q_heads);
    const int hk = h / group, g = h % group;
    drow = ((long long)(b * num_kv_heads + hk) * num_q_blocks + qb) * (group * R) + g * R + r;
    dhi = q_hi;
    dlo = q_lo;
    n_read = rows = q_sub;
  } else {
    const long long kv = w - n_qvec;
    if (kv >= n_kvec) return;
    const int t = (int)(kv % T);
    long long r = kv / T;
    const int p = (int)(r % num_pages);
    r /= num_pages;
    const int hk = (int)(r % num_kv_heads);
    const int b = (int)(r / num_kv_heads);
    const int phys = page_table[(long long)b * pages_per_seq + p];
    n_read = rows = k_sub;
    if (phys < 0 || phys >= num_phys_pages) {  // outside the pool: reported, not read
      if (lane == 0) set_status(COSA_ERR_INVALID_ARG);
      n_read = 0;  // the pooled vector is written as zero
      src = k_pool;
    } else {
      src = k_pool + (((long long)phys * num_kv_heads + hk) * page_size + (long long)t * k_sub) * D;
    }
    drow = kv;
    dhi = k_hi;
    dlo = k_lo;
  }
  const int c = lane % LPR;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 4
  for (int r = lane / LPR; r < n_read; r += RPI) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (long long)r * D) + c);
    const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(hh[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
  }
  if (lane < LPR) {
    const float inv = 1.0f / (float)rows;  // rows is a power of two: exact
    float hi[8], lo[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float x = acc[i] * inv;
      hi[i] = to_tf32(x);
      lo[i] = to_tf32(x - hi[i]);
    }
    float4* ph = reinterpret_cast<float4*>(dhi + drow * D) + 2 * c;
    float4* pl = reinterpret_cast<float4*>(dlo + drow * D) + 2 * c;
    ph[0] = make_float4(hi[0], hi[1], hi[2], hi[3]);
    ph[1] = make_float4(hi[4], hi[5], hi[6], hi[7]);
    pl[0] = make_float4(lo[0], lo[1], lo[2], lo[3]);
    pl[1] = make_float4(lo[4], lo[5], lo[6], lo[7]);
  }
}

// ---------------------------------------------------------------------------
// KAP pooling fused into the prefill's write of its attention inputs.  The Q, K and
// V a prefill layer produces arrive token-major ([B][N][H][D], the projection's
// layout); attention reads Q head-major and K / V from the paged cache.  This kernel
// does that write (Q relaid head-major, K and V scattered into their pages through
// the page table) and, in the same pass over the rows, the downsampling of
// kap_pool_kernel, so Stage 1 needs no second read of Q and K (cosa_kap_rank then
// finishes it from the workspace).  Work items are those of kap_pool_kernel; a key
// item also copies the V rows of its token range.  Each lane accumulates the same
// rows in the same order as kap_pool_kernel, so the pooled vectors are identical.
// With pooling off (q_hi null) it is the plain write.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) prefill_write_kernel(
    const __nv_bfloat16* __restrict__ q_tok, const __nv_bfloat16* __restrict__ k_tok,
    const __nv_bfloat16* __restrict__ v_tok, const int32_t* __restrict__ page_table,
    __nv_bfloat16* __restrict__ q_out, __nv_bfloat16* __restrict__ k_pool,
    __nv_bfloat16* __restrict__ v_pool, float* __restrict__ q_hi, float* __restrict__ q_lo,
    float* __restrict__ k_hi, float* __restrict__ k_lo, long long n_qvec, int q_sub,
    long long n_kvec, int k_sub, int num_q_heads, int num_kv_heads, int group, int R,
    int num_q_blocks, int page_size, int num_pages, int pages_per_seq, int num_phys_pages,
    int T, int seq_len) {
  constexpr int LPR = D / 8;     // lanes per row: each lane moves 8 bf16 (16 B)
  constexpr int RPI = 32 / LPR;  // rows covered per warp-wide load
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const bool pool = q_hi != nullptr;
  const __nv_bfloat16* src;
  const __nv_bfloat16* vsrc = nullptr;
  __nv_bfloat16* dst;
  __nv_bfloat16* vdst = nullptr;
  long long src_stride, drow;
  float *dhi, *dlo;
  int rows;
  if (w < n_qvec) {
    const int r = (int)(w % R);
    long long t1 = w / R;
    const int qb = (int)(t1 % num_q_blocks);
    const long long bhq = t1 / num_q_blocks;
    const int h = (int)(bhq % num_q_heads);
    const int b = (int)(bhq / num_q_heads);
    const int hk = h / group, g = h % group;
    const long long tok0 = (long long)qb * (R * q_sub) + (long long)r * q_sub;
    src = q_tok + (((long long)b * seq_len + tok0) * num_q_heads + h) * D;
    src_stride = (long long)num_q_heads * D;
    dst = q_out + (bhq * seq_len + tok0) * D;
    drow = ((long long)(b * num_kv_heads + hk) * num_q_blocks + qb) * (group * R) + g * R + r;
    dhi = q_hi;
    dlo = q_lo;
    rows = q_sub;
  } else {
    const long long kv = w - n_qvec;
    if (kv >= n_kvec) return;
    const int t = (int)(kv % T);
    long long r = kv / T;
    const int p = (int)(r % num_pages);
    r /= num_pages;
    const int hk = (int)(r % num_kv_heads);
    const int b = (int)(r / num_kv_heads);
    const int phys = page_table[(long long)b * pages_per_seq + p];
    const long long tok0 = (long long)p * page_size + (long long)t * k_sub;
    const long long off_src = (((long long)b * seq_len + tok0) * num_kv_heads + hk) * D;
    src = k_tok + off_src;
    vsrc = v_tok + off_src;
    src_stride = (long long)num_kv_heads * D;
    if (phys < 0 || phys >= num_phys_pages) {  // outside the pool: reported, not written
      if (lane == 0) set_status(COSA_ERR_INVALID_ARG);
      dst = nullptr;  // the pooled vector still comes from the rows read
    } else {
      const long long off_dst =
          (((long long)phys * num_kv_heads + hk) * page_size + (long long)t * k_sub) * D;
      dst = k_pool + off_dst;
      vdst = v_pool + off_dst;
    }
    drow = kv;
    dhi = k_hi;
    dlo = k_lo;
    rows = k_sub;
  }
  const int c = lane % LPR;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  // one loop per case (Q rows; K and V rows; K rows of a page outside the pool, pooled
  // only), so no loop carries a branch per row
  auto rows_loop = [&](auto copy_k, auto copy_v) {
    constexpr bool CK = decltype(copy_k)::value, CV = decltype(copy_v)::value;
#pragma unroll 4
    for (int r = lane / LPR; r < rows; r += RPI) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (long long)r * src_stride) + c);
      if (CK) reinterpret_cast<uint4*>(dst + (long long)r * D)[c] = v;
      if (CV) {
        const uint4 vv = __ldg(reinterpret_cast<const uint4*>(vsrc + (long long)r * src_stride) + c);
        reinterpret_cast<uint4*>(vdst + (long long)r * D)[c] = vv;
      }
      const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(hh[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
  };
  if (vdst) rows_loop(std::true_type(), std::true_type());
  else if (dst) rows_loop(std::true_type(), std::false_type());
  else rows_loop(std::false_type(), std::false_type());
  if (!pool) return;
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
  }
  if (lane < LPR) {
    const float inv = 1.0f / (float)rows;  // rows is a power of two: exact
    float hi[8], lo[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float x = acc[i] * inv;
      hi[i] = to_tf32(x);
      lo[i] = to_tf32(x - hi[i]);
    }
    float4* ph = reinterpret_cast<float4*>(dhi + drow * D) + 2 * c;
    float4* pl = reinterpret_cast<float4*>(dlo + drow * D) + 2 * c;
    ph[0] = make_float4(hi[0], hi[1], hi[2], hi[3]);
    ph[1] = make_float4(hi[4], hi[5], hi[6], hi[7]);
    pl[0] = make_float4(lo[0], lo[1], lo[2], lo[3]);
    pl[1] = make_float4(lo[4], lo[5], lo[6], lo[7]);
  }
}

// ---------------------------------------------------------------------------
// K3: MaxNorm + HRM (from the page maxima) or caller-given scores, then
// selection + ordering.  grid.x = nQB (heaviest first), grid.y = B * H_q, or
// B * H_kv in group mode: one list for the G query heads of a KV head, from
// S[p] = max over the heads of each head's MaxNorm score and HRM[p] = any head's
// flag (the group-shared selection; the pages describe per-head selection only).
// key = hrm << 63 | float_bits(S) << 31 | (2^31 - 1 - page): larger is better.
// ---------------------------------------------------------------------------
constexpr int ORDER_THREADS = 512;

__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  if (total) *total = warp_sums[nw - 1];
  __syncthreads();
  return before;
}

// Descending bitonic sort of 32 E 64-bit keys held by one warp: element e = 32 i + lane
// in x[i].  Pairs 32 or more apart sit in one lane's registers; the others are exchanged
// between lanes.  Fully unrolled, so every register index is a constant.
template <int E>
__device__ __forceinline__ void warp_sort_desc(unsigned long long (&x)[E]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int kk = 2; kk <= 32 * E; kk <<= 1) {
#pragma unroll
    for (int j = kk >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
        const int jj = j >> 5;
#pragma unroll
        for (int i = 0; i < E; ++i) {
          if ((i ^ jj) > i) {
            const int e = 32 * i + lane;
            const unsigned long long a = x[i], b = x[i ^ jj];
            const bool desc = (e & kk) == 0;  // larger first in this block
            const bool sw = desc ? (a < b) : (a > b);
            x[i] = sw ? b : a;
            x[i ^ jj] = sw ? a : b;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const int e = 32 * i + lane;
          const unsigned long long y = __shfl_xor_sync(0xffffffffu, x[i], j);
          const bool keep_max = ((e & j) == 0) == ((e & kk) == 0);
          x[i] = keep_max ? (x[i] > y ? x[i] : y) : (x[i] < y ? x[i] : y);
        }
      }
    }
  }
}

struct KapPageMax {
  const float* a;       // triangular page maxima (see kap_tc.cuh)
  const float* row_max; // [B * H_kv * nQB * G * R]
  const int* row_arg;   // first page attaining it
  int num_kv_heads, group, R;
};

constexpr int ORDER_MAX_ROWS = 64;  // representative rows read by one CTA (G * R in group mode)

// RT: representatives per q-block and head (q_block / q_sub) fixed at compile time, so the
// per-page loop over them carries no dead iterations; 0 where the scores come given
template <bool FROM_A, bool GROUP, int RT>
__global__ void __launch_bounds__(ORDER_THREADS, 3) kap_order_kernel(
    const float* __restrict__ scores, const uint8_t* __restrict__ hrm, KapPageMax pm,
    float* __restrict__ scores_out, uint8_t* __restrict__ hrm_out, int32_t* __restrict__ order,
    int32_t* __restrict__ count, int num_q_heads, int num_q_blocks, int num_pages, int q_block,
    int page_size, float budget, int sink, int ascending, int k_cap) {
  extern __shared__ unsigned long long keys[];  // [npow2] by page, then max(npow2, 32) kept keys
  __shared__ int warp_sums[32];
  __shared__ int hist_s[256];
  __shared__ int sel_s[3];
  __shared__ float m_s[ORDER_MAX_ROWS];
  __shared__ int arg_s[ORDER_MAX_ROWS];
  const int qb = num_q_blocks - 1 - blockIdx.x;
  const int bhq = blockIdx.y;
  const long long row = (long long)bhq * num_q_blocks + qb;
  const int n_b = causal_pages(qb, q_block, page_size);
  const int first_diag = (qb * q_block) / page_size;
  const int n_f = forced_count(qb, q_block, page_size, sink);
  const int k_b = budget_count(qb, q_block, page_size, sink, budget);
  const int quota = k_b - n_f;
  int npow2 = 1;
  while (npow2 < n_b) npow2 <<= 1;

  const float* arow = nullptr;
  const int n_heads = GROUP ? pm.group : 1;  // heads whose rows this CTA reads
  if (FROM_A) {
    int b, hk, g;
    if (GROUP) {
      b = bhq / pm.num_kv_heads;
      hk = bhq % pm.num_kv_heads;
      g = 0;
    } else {
      b = bhq / num_q_heads;
      const int h = bhq % num_q_heads;
      hk = h / pm.group;
      g = h % pm.group;
    }
    const int GR = pm.group * pm.R;
    const long long slab = (long long)b * pm.num_kv_heads + hk;
    const long long rep0 = (slab * num_q_blocks + qb) * GR + (long long)g * pm.R;
    arow = pm.a + slab * GR * cum_pages(num_q_blocks, q_block, page_size) +
           (long long)GR * cum_pages(qb, q_block, page_size) + (long long)g * pm.R * n_b;
    for (int t = threadIdx.x; t < n_heads * pm.R; t += blockDim.x) {
      m_s[t] = pm.row_max[rep0 + t];
      arg_s[t] = pm.row_arg[rep0 + t];
    }
    __syncthreads();
  }
  // (one head's row maxima and first maximal pages, in registers)
  constexpr int RM = RT > 0 ? RT : 1;
  float m_r[RM];
  int arg_r[RM];
#pragma unroll
  for (int i = 0; i < RM; ++i) {
    m_r[i] = FROM_A && !GROUP ? m_s[i] : 0.f;
    arg_r[i] = FROM_A && !GROUP ? arg_s[i] : -1;
  }
  const float* srow = FROM_A ? nullptr : scores + row * num_pages;
  const uint8_t* hrow = FROM_A ? nullptr : hrm + row * num_pages;
  const float invR = FROM_A ? 1.0f / (float)pm.R : 0.f;  // R is a power of two
  for (int p = threadIdx.x; p < npow2; p += blockDim.x) {
    unsigned long long key = 0ull;
    if (p < n_b) {
      float sv;
      int flag;
      if (FROM_A) {
        // MaxNorm: S[p] = mean_r exp(a[r][p] - m_r); HRM: p is some row's first
        // maximum (group mode: the largest head score, any head's flag).  A head's
        // R <= 8 page maxima are loaded together, then summed in row order.
        sv = 0.f;
        flag = 0;
        for (int g = 0; g < n_heads; ++g) {
          float av[RM];
#pragma unroll
          for (int i = 0; i < RM; ++i) av[i] = arow[(long long)(g * RM + i) * n_b + p];
          float sg = 0.f;
#pragma unroll
          for (int i = 0; i < RM; ++i) {
            const int r = g * RM + i;
            sg += expf(av[i] - (GROUP ? m_s[r] : m_r[i]));
            flag |= ((GROUP ? arg_s[r] : arg_r[i]) == p);
          }
          sv = fmaxf(sv, sg * invR);
        }
      } else {
        sv = srow[p];
        flag = hrow[p] != 0;
      }
      if (scores_out) scores_out[row * num_pages + p] = sv;
      if (hrm_out) hrm_out[row * num_pages + p] = (uint8_t)flag;
      unsigned long long bits = (unsigned long long)__float_as_uint(sv);
      key = ((unsigned long long)(flag != 0) << 63) | (bits << 31) |
            (unsigned long long)(0x7fffffff - p);
    }
    keys[p] = key;
  }
  if (scores_out || hrm_out)
    for (int p = n_b + threadIdx.x; p < num_pages; p += blockDim.x) {
      if (scores_out) scores_out[row * num_pages + p] = 0.f;
      if (hrm_out) hrm_out[row * num_pages + p] = 0;
    }
  __syncthreads();
  // ---- threshold: the quota-th largest key among the pages that are not forced,
  // by radix select over 8-bit digits (keys are unique: the page is in the low bits).
  // Selected = forced pages + non-forced pages with (key >> thr_shift) >= thr_prefix.
  const int n_nf = n_b - n_f;
  unsigned long long thr_prefix = 0ull;
  int thr_shift = 64;  // 64: no non-forced page (quota <= 0); -1: every one
  if (quota >= n_nf) {
    thr_shift = -1;
  } else if (quota > 0) {
    int r = quota;  // rank (1 = largest) still to find inside the current bucket
    unsigned long long prefix = 0ull;
    for (int shift = 56;; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += blockDim.x) hist_s[i] = 0;
      __syncthreads();
      for (int p0 = 0; p0 < n_b; p0 += blockDim.x) {
        const int p = p0 + threadIdx.x;
        int bin = -1;
        if (p < n_b && !(p < sink || p >= first_diag)) {
          const unsigned long long key = keys[p];
          if (shift == 56 || (key >> (shift + 8)) == prefix) bin = (int)((key >> shift) & 255ull);
        }
        // warp-aggregated: many keys share their leading digits
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist_s[bin], __popc(peers));
      }
      __syncthreads();
      if (threadIdx.x < 32) {
        // lane l holds bins 255 - 8 l ... 248 - 8 l (largest digits first)
        const int lane = threadIdx.x;
        int c[8], sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          c[e] = hist_s[255 - 8 * lane - e];
          sum += c[e];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int run = incl - sum;
        if (run < r && r <= incl) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (run + c[e] >= r) {
              sel_s[0] = 255 - 8 * lane - e;  // the digit holding rank r
              sel_s[1] = r - run;             // its rank inside that digit
              sel_s[2] = c[e];                // keys with that digit
              break;
            }
            run += c[e];
          }
        }
      }
      __syncthreads();
      const int bin = sel_s[0];
      r = sel_s[1];
      prefix = (prefix << 8) | (unsigned long long)bin;
      if (sel_s[2] == r || shift == 0) {  // the whole digit is taken, or the key is exact
        thr_prefix = prefix;
        thr_shift = shift;
        break;
      }
      __syncthreads();
    }
  }
  auto selected = [&](int p) -> bool {
    if (p < sink || p >= first_diag) return true;
    if (thr_shift < 0) return true;
    if (thr_shift >= 64) return false;
    return (keys[p] >> thr_shift) >= thr_prefix;
  };
  // ---- compaction in page order (contiguous chunks per thread)
  const int per = (n_b + blockDim.x - 1) / blockDim.x;
  const int beg = threadIdx.x * per;
  int sel_local = 0;
  for (int p = beg; p < beg + per && p < n_b; ++p) sel_local += selected(p);
  int total = 0;
  int pos = block_excl_scan(sel_local, warp_sums, &total);
  int32_t* orow = order + row * k_cap;
  if (ascending) {
    for (int p = beg; p < beg + per && p < n_b; ++p)
      if (selected(p)) orow[pos++] = p;
  } else {
    // kept keys only, then a sort (descending) of those
    unsigned long long* kept = keys + npow2;
    int m = 1;
    while (m < total) m <<= 1;
    for (int p = beg; p < beg + per && p < n_b; ++p)
      if (selected(p)) kept[pos++] = keys[p];
    if (total <= 32 * (int)(blockDim.x >> 5)) {
      // up to one run of 32 keys per warp: each warp sorts its run in registers, then
      // each key's place is its place in its run plus, for every other run, the
      // number of that run's keys above it (a binary search: runs are descending, and
      // the zero keys that pad the last run lie below every key)
      const int lane = (int)threadIdx.x & 31, warp = (int)threadIdx.x >> 5;
      const int runs = (total + 31) >> 5;
      __syncthreads();
      if (warp < runs) {
        const int e = 32 * warp + lane;
        unsigned long long x[1] = {e < total ? kept[e] : 0ull};
        warp_sort_desc<1>(x);
        kept[e] = x[0];
      }
      __syncthreads();
      if ((int)threadIdx.x < total) {
        const int t = (int)threadIdx.x, own = t >> 5;
        const unsigned long long mine = kept[t];
        int rank = t & 31;
        for (int r = 0; r < runs; ++r) {
          if (r == own) continue;
          const unsigned long long* run = kept + 32 * r;
          int lo = 0, hi = 32;  // first index whose key is not above mine
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (run[mid] > mine) lo = mid + 1;
            else hi = mid;
          }
          rank += lo;
        }
        orow[rank] = 0x7fffffff - (int)(mine & 0x7fffffffull);
      }
    } else {
      const int mw = m < 32 ? 32 : m;  // whole warps take part in the register stages
      for (int i = total + threadIdx.x; i < mw; i += blockDim.x) kept[i] = 0ull;  // below every key
      __syncthreads();
      // Bitonic sort, descending.  Stages pairing elements 32 or more apart go through
      // shared memory; the others pair lanes of one warp and run in registers (element i
      // is held by lane i % 32 of its warp; the partner of i is i ^ j).
      auto warp_stages = [&](int k_lo, int k_hi) {
        for (int i0 = 0; i0 < mw; i0 += blockDim.x) {
          const int i = i0 + (int)threadIdx.x;
          if (i >= mw) continue;  // whole warps: mw and blockDim are multiples of 32
          unsigned long long x = kept[i];
          for (int kk = k_lo; kk <= k_hi; kk <<= 1)
            for (int j = (kk >> 1) < 16 ? (kk >> 1) : 16; j > 0; j >>= 1) {
              const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j);
              const bool keep_max = ((i & j) == 0) == ((i & kk) == 0);
              x = keep_max ? (x > y ? x : y) : (x < y ? x : y);
            }
          kept[i] = x;
        }
        __syncthreads();
      };
      if (m >= 2) warp_stages(2, m < 32 ? m : 32);  // every size up to 32 at once
      for (int kk = 64; kk <= m; kk <<= 1) {
        for (int j = kk >> 1; j >= 32; j >>= 1) {
          for (int i = threadIdx.x; i < m; i += blockDim.x) {
            const int ixj = i ^ j;
            if (ixj > i) {
              const unsigned long long x = kept[i], y = kept[ixj];
              const bool desc = (i & kk) == 0;
              if (desc ? (x < y) : (x > y)) { kept[i] = y; kept[ixj] = x; }
            }
          }
          __syncthreads();
        }
        warp_stages(kk, kk);
      }
      for (int i = threadIdx.x; i < total; i += blockDim.x)
        orow[i] = 0x7fffffff - (int)(kept[i] & 0x7fffffffull);
    }
  }
  for (int j = total + threadIdx.x; j < k_cap; j += blockDim.x) orow[j] = -1;
  if (threadIdx.x == 0) {
    count[row] = total;
    if (total != k_b) set_status(COSA_ERR_INVALID_ARG);  // cannot happen for valid shapes
  }
}

// ---------------------------------------------------------------------------
// Proxy-bound pre-skip (a variant the pages do not give; off unless asked).  The
// pages' in-kernel skip (gist.science/pt §2.3 "Saltado no Kernel") still costs every
// listed page its K load and QK^T.  This filter applies the same kind of test one
// stage earlier, on the proxy's page maxima a[r][p] and the proxy's own running max
// along the ordered list, and removes the pages it rejects before the kernel runs:
//   ahat_r(j) = max over list positions j' < j of a[r][p_j'];
//   representative r keeps position j iff a[r][p_j] > -inf and (ahat_r(j) = -inf
//     or (a[r][p_j] + margin) - ahat_r(j) >= ln eps);
//   position j >= 1 is removed iff no representative keeps it.
// One CTA per (b, h_q, q-block): the list is read into shared memory, each thread
// takes a contiguous run of positions, the runs' maxima are scanned per
// representative (one warp per representative), each thread then walks its run,
// and the survivors are written back in list order (-1 after them).
// ---------------------------------------------------------------------------
constexpr int PRESKIP_THREADS = 256;
constexpr int PRESKIP_MAX_R = 8;

__global__ void __launch_bounds__(PRESKIP_THREADS) kap_preskip_kernel(
    KapPageMax pm, int32_t* __restrict__ order, int32_t* __restrict__ count,
    uint8_t* __restrict__ skip_log, int num_q_heads, int num_q_blocks, int q_block,
    int page_size, int k_cap, float log_eps, float margin) {
  extern __shared__ int lst[];  // [k_cap] the list, as read
  __shared__ float run_max[PRESKIP_THREADS][PRESKIP_MAX_R];  // per run, then exclusive scan
  __shared__ int warp_sums[32];
  const int qb = blockIdx.x, bhq = blockIdx.y;
  const long long row = (long long)bhq * num_q_blocks + qb;
  const int n_b = causal_pages(qb, q_block, page_size);
  const int R = pm.R;
  const int b = bhq / num_q_heads, h = bhq % num_q_heads;
  const int hk = h / pm.group, g = h % pm.group;
  const int GR = pm.group * R;
  const long long slab = (long long)b * pm.num_kv_heads + hk;
  const float* arow = pm.a + slab * GR * cum_pages(num_q_blocks, q_block, page_size) +
                      (long long)GR * cum_pages(qb, q_block, page_size) + (long long)g * R * n_b;
  int32_t* orow = order + row * k_cap;
  const int n = min(max(count[row], 0), k_cap);
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const int p = orow[j];
    lst[j] = (p >= 0 && p < n_b) ? p : -1;  // out-of-range ids are flagged below
  }
  __syncthreads();
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int j0 = min(n, (int)threadIdx.x * per), j1 = min(n, j0 + per);
  int bad = 0;
  float rm[PRESKIP_MAX_R];
#pragma unroll
  for (int r = 0; r < PRESKIP_MAX_R; ++r) rm[r] = -INFINITY;
  for (int j = j0; j < j1; ++j) {
    const int p = lst[j];
    if (p < 0) { bad = 1; continue; }
#pragma unroll
    for (int r = 0; r < PRESKIP_MAX_R; ++r)
      if (r < R) rm[r] = fmaxf(rm[r], __ldg(arow + (long long)r * n_b + p));
  }
#pragma unroll
  for (int r = 0; r < PRESKIP_MAX_R; ++r) run_max[threadIdx.x][r] = rm[r];
  if (__syncthreads_or(bad)) {  // not a list of this block's causal pages: left as is
    if (threadIdx.x == 0) set_status(COSA_ERR_INVALID_ARG);
    return;
  }
  // exclusive max-scan of the runs' maxima, warp r for representative r
  {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int PL = PRESKIP_THREADS / 32;  // runs per lane
    if (warp < R) {
      float loc = -INFINITY;
#pragma unroll
      for (int i = 0; i < PL; ++i) loc = fmaxf(loc, run_max[lane * PL + i][warp]);
      float inc = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc = fmaxf(inc, y);
      }
      float run = __shfl_up_sync(0xffffffffu, inc, 1);  // max over the lanes before
      if (lane == 0) run = -INFINITY;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        const float v = run_max[lane * PL + i][warp];
        run_max[lane * PL + i][warp] = run;
        run = fmaxf(run, v);
      }
    }
  }
  __syncthreads();
  // walk this thread's run: decisions, then the survivors' positions
  float ahat[PRESKIP_MAX_R];
#pragma unroll
  for (int r = 0; r < PRESKIP_MAX_R; ++r) ahat[r] = run_max[threadIdx.x][r];
  uint32_t keep_bits = 0;  // per = ceil(n / 256) <= 32 positions per thread (n <= 8192)
  int kept = 0;
  for (int j = j0; j < j1; ++j) {
    const int p = lst[j];
    bool keep = j == 0;
#pragma unroll
    for (int r = 0; r < PRESKIP_MAX_R; ++r) {
      if (r >= R) break;
      const float v = __ldg(arow + (long long)r * n_b + p);
      if (v != -INFINITY && (ahat[r] == -INFINITY || (v + margin) - ahat[r] >= log_eps)) keep = true;
      ahat[r] = fmaxf(ahat[r], v);
    }
    if (keep) {
      keep_bits |= 1u << (j - j0);
      ++kept;
    }
    if (skip_log) skip_log[row * k_cap + j] = keep ? 0 : 1;
  }
  int total = 0;
  int pos = block_excl_scan(kept, warp_sums, &total);
  for (int j = j0; j < j1; ++j)
    if (keep_bits >> (j - j0) & 1u) orow[pos++] = lst[j];
  for (int j = total + threadIdx.x; j < k_cap; j += blockDim.x) orow[j] = -1;
  if (threadIdx.x == 0) count[row] = total;
}

}  // namespace cosa
