// Stage 1 of CoSA, the Kernel-Aware Proxy (gist.science/pt, "CoSA" technical
// summary, §2.2 "Estágio 1: Kernel-Aware Proxy (KAP)").
//
//   kap_pool_kernel   query / key downsampling ("Ranking de Blocos"): mean of
//                     q_sub consecutive query rows and of k_sub consecutive keys
//                     of each logical page (read through the page table).
//                     HBM-bound: one warp per pooled vector, 16-byte loads.
//   kap_score_kernel  approximate scores, MaxPool over each page's sub-keys,
//                     MaxNorm per representative row, HRM flags ("Geração de
//                     Flag HRM").  One CTA per (q-block, batch, KV head, head
//                     group); the pooled keys of the KV head are streamed
//                     from L2 and shared by all representatives of the group.
//   kap_order_kernel  budgeted selection and the computation-order mask
//                     ("Ordenação por Grupo de Flags"): packed 64-bit rank keys,
//                     block bitonic sort, forced pages kept, scan-compaction.
#pragma once

#include "common.cuh"

namespace cosa {

// ---------------------------------------------------------------------------
// K1: pooling.  Work item w < n_qvec: pooled query vector w of the flattened
// [B][H_q][N / q_sub] index; else pooled key vector (w - n_qvec) of the
// [B][H_kv][nP][T] index.  Output rows are fp32 [.][D].
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) kap_pool_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_pool,
    const int32_t* __restrict__ page_table, float* __restrict__ qhat, float* __restrict__ khatT,
    long long n_qvec, int q_sub, long long n_kvec, int k_sub, int num_kv_heads, int page_size,
    int num_pages, int pages_per_seq, int T, int khat_stride) {
  constexpr int LPR = D / 8;   // lanes per row: each lane loads 8 bf16 (16 B)
  constexpr int RPI = 32 / LPR;  // rows covered per warp-wide load
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const __nv_bfloat16* src;
  float* dst;
  long long dst_stride;  // distance between consecutive d of the output vector
  int rows;
  if (w < n_qvec) {
    src = q + w * (long long)q_sub * D;
    dst = qhat + w * D;
    dst_stride = 1;
    rows = q_sub;
  } else {
    long long kv = w - n_qvec;
    if (kv >= n_kvec) return;
    int t = (int)(kv % T);
    long long r = kv / T;
    int p = (int)(r % num_pages);
    r /= num_pages;
    int hk = (int)(r % num_kv_heads);
    int b = (int)(r / num_kv_heads);
    int phys = page_table[(long long)b * pages_per_seq + p];
    src = k_pool + (((long long)phys * num_kv_heads + hk) * page_size + (long long)t * k_sub) * D;
    // transposed: khatT[b][hk][d][khat_stride], sub-key index p * T + t
    dst = khatT + ((long long)(b * num_kv_heads + hk) * D) * khat_stride + (long long)p * T + t;
    dst_stride = khat_stride;
    rows = k_sub;
  }
  const int c = lane % LPR;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 4
  for (int r = lane / LPR; r < rows; r += RPI) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (long long)r * D) + c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
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
    if (dst_stride == 1) {
      float4 o0 = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      float4 o1 = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      reinterpret_cast<float4*>(dst)[2 * c] = o0;
      reinterpret_cast<float4*>(dst)[2 * c + 1] = o1;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[(long long)(c * 8 + i) * dst_stride] = acc[i] * inv;
    }
  }
}

// ---------------------------------------------------------------------------
// K2: scores, MaxPool, MaxNorm, HRM.
// grid.x = nQB (heaviest q-block first), grid.y = B * H_kv * head_groups.
// The NR = hpc * R representatives of the CTA's heads sit in shared memory as
// qT[d][rep]; each thread owns 4 consecutive sub-keys and computes their full
// dot products with every representative (an NR x 4 register tile), reading
// the pooled keys from the transposed layout khatT[d][sub-key] so that one
// warp load is one contiguous 512-byte row.  a[rep][page] stays in shared
// memory until the row maxima are known.
// ---------------------------------------------------------------------------
constexpr int SCORE_THREADS = 256;

template <int D, int NRMAX>
__global__ void __launch_bounds__(SCORE_THREADS) kap_score_kernel(
    const float* __restrict__ qhat, const float* __restrict__ khatT, float* __restrict__ scores,
    uint8_t* __restrict__ hrm_out, int num_q_heads, int num_kv_heads, int group, int hpc,
    int num_q_blocks, int num_pages, int khat_stride, int R, int T, int q_sub, int k_sub,
    int page_size, int q_block, float scale) {
  extern __shared__ float smem[];
  const int NR = hpc * R;
  float* qT = smem;                   // [D][NRMAX]
  float* a_s = qT + D * NRMAX;        // [NR][num_pages]
  __shared__ float m_s[NRMAX];
  __shared__ int arg_s[NRMAX];

  const int qb = num_q_blocks - 1 - blockIdx.x;
  const int head_groups = group / hpc;
  const int hg = blockIdx.y % head_groups;
  const int hk = (blockIdx.y / head_groups) % num_kv_heads;
  const int b = blockIdx.y / (head_groups * num_kv_heads);
  const int h0 = hk * group + hg * hpc;
  const int n_b = causal_pages(qb, q_block, page_size);
  const int tid = threadIdx.x;

  for (int i = tid; i < NRMAX * D; i += blockDim.x) {
    const int rep = i % NRMAX, d = i / NRMAX;
    float v = 0.f;
    if (rep < NR) {
      const int hh = rep / R, r = rep % R;
      v = qhat[(((long long)(b * num_q_heads + h0 + hh) * num_q_blocks + qb) * R + r) * D + d];
    }
    qT[d * NRMAX + rep] = v;
  }
  __syncthreads();

  const int ns = n_b * T;             // causal sub-keys
  const int nq = (ns + 3) >> 2;       // quads of sub-keys
  const float* kb = khatT + (long long)(b * num_kv_heads + hk) * D * khat_stride;
  for (int base = 0; base < nq; base += blockDim.x) {
    const int qd = base + tid;
    const bool valid = qd < nq;
    const int s0 = qd * 4;
    float acc[NRMAX][4];
#pragma unroll
    for (int r = 0; r < NRMAX; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
    if (valid) {
      const float* kp = kb + s0;
#pragma unroll 8
      for (int d = 0; d < D; ++d) {
        const float4 kv = __ldg(reinterpret_cast<const float4*>(kp + (long long)d * khat_stride));
        const float* qrow = qT + d * NRMAX;
#pragma unroll
        for (int r4 = 0; r4 < NRMAX / 4; ++r4) {
          if (r4 * 4 < NR) {
            const float4 qv = *reinterpret_cast<const float4*>(qrow + r4 * 4);
            const float qq[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc[r4 * 4 + e][0] = fmaf(qq[e], kv.x, acc[r4 * 4 + e][0]);
              acc[r4 * 4 + e][1] = fmaf(qq[e], kv.y, acc[r4 * 4 + e][1]);
              acc[r4 * 4 + e][2] = fmaf(qq[e], kv.z, acc[r4 * 4 + e][2]);
              acc[r4 * 4 + e][3] = fmaf(qq[e], kv.w, acc[r4 * 4 + e][3]);
            }
          }
        }
      }
    }
    // causal visibility per (rep, sub-key), then MaxPool over each page's sub-keys
    int first_tok[4], page_of[4];
    bool in_range[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sidx = s0 + u;
      page_of[u] = sidx / T;
      first_tok[u] = page_of[u] * page_size + (sidx % T) * k_sub;
      in_range[u] = valid && sidx < ns;
    }
#pragma unroll
    for (int r = 0; r < NRMAX; ++r) {
      if (r < NR) {
        const int rep_last = qb * q_block + ((r % R) + 1) * q_sub - 1;
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          v[u] = (in_range[u] && first_tok[u] <= rep_last) ? acc[r][u] * scale : -INFINITY;
        if (T >= 4) {  // all four sub-keys belong to one page
          float m = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
          if (T == 8) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
          if (valid && (T == 4 || (qd & 1) == 0)) a_s[r * num_pages + page_of[0]] = m;
        } else if (T == 2) {
          if (in_range[0]) a_s[r * num_pages + page_of[0]] = fmaxf(v[0], v[1]);
          if (in_range[2]) a_s[r * num_pages + page_of[2]] = fmaxf(v[2], v[3]);
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (in_range[u]) a_s[r * num_pages + page_of[u]] = v[u];
        }
      }
    }
  }
  __syncthreads();

  // row max and first page holding it, per representative
  const int warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
  for (int r = warp; r < NR; r += nwarps) {
    float m = -INFINITY;
    for (int p = lane; p < n_b; p += 32) m = fmaxf(m, a_s[r * num_pages + p]);
    m = warp_max(m);
    int first = 0x7fffffff;
    for (int p = lane; p < n_b; p += 32)
      if (a_s[r * num_pages + p] == m) { first = p; break; }
    first = warp_min_int(first);
    if (lane == 0) { m_s[r] = m; arg_s[r] = first; }
  }
  __syncthreads();

  // S[p] = mean_r exp(a[r][p] - m_r); HRM[p] = p is some row's first maximum
  const float invR = 1.0f / (float)R;  // R is a power of two
  for (int i = tid; i < hpc * num_pages; i += blockDim.x) {
    const int hh = i / num_pages, p = i % num_pages;
    float sv = 0.f;
    int flag = 0;
    if (p < n_b) {
      for (int r = 0; r < R; ++r) {
        const int rep = hh * R + r;
        sv += expf(a_s[rep * num_pages + p] - m_s[rep]);
        flag |= (arg_s[rep] == p);
      }
      sv *= invR;
    }
    const long long o = ((long long)(b * num_q_heads + h0 + hh) * num_q_blocks + qb) * num_pages + p;
    scores[o] = sv;
    hrm_out[o] = (uint8_t)flag;
  }
}

// ---------------------------------------------------------------------------
// K3: selection + ordering.  grid.x = nQB (heaviest first), grid.y = B * H_q.
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

__global__ void __launch_bounds__(ORDER_THREADS) kap_order_kernel(
    const float* __restrict__ scores, const uint8_t* __restrict__ hrm, int32_t* __restrict__ order,
    int32_t* __restrict__ count, int num_q_blocks, int num_pages, int q_block, int page_size,
    float budget, int sink, int ascending, int k_cap) {
  extern __shared__ unsigned long long keys[];  // [npow2]
  __shared__ int warp_sums[32];
  const int qb = num_q_blocks - 1 - blockIdx.x;
  const long long row = (long long)blockIdx.y * num_q_blocks + qb;
  const int n_b = causal_pages(qb, q_block, page_size);
  const int first_diag = (qb * q_block) / page_size;
  const int n_f = forced_count(qb, q_block, page_size, sink);
  const int k_b = budget_count(qb, q_block, page_size, sink, budget);
  const int quota = k_b - n_f;
  int npow2 = 1;
  while (npow2 < n_b) npow2 <<= 1;
  const float* srow = scores + row * num_pages;
  const uint8_t* hrow = hrm + row * num_pages;
  for (int p = threadIdx.x; p < npow2; p += blockDim.x) {
    unsigned long long key = 0ull;
    if (p < n_b) {
      unsigned long long bits = (unsigned long long)__float_as_uint(srow[p]);
      key = ((unsigned long long)(hrow[p] != 0) << 63) | (bits << 31) |
            (unsigned long long)(0x7fffffff - p);
    }
    keys[p] = key;
  }
  __syncthreads();
  // bitonic sort, descending
  for (int kk = 2; kk <= npow2; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < npow2; i += blockDim.x) {
        int ixj = i ^ j;
        if (ixj > i) {
          unsigned long long a = keys[i], c = keys[ixj];
          bool desc = (i & kk) == 0;
          if (desc ? (a < c) : (a > c)) { keys[i] = c; keys[ixj] = a; }
        }
      }
      __syncthreads();
    }
  }
  // selection over the sorted list: forced pages always, others while quota lasts
  const int per = (npow2 + blockDim.x - 1) / blockDim.x;
  const int beg = threadIdx.x * per;
  int nf_local = 0;
  for (int i = beg; i < beg + per && i < n_b; ++i) {
    int page = 0x7fffffff - (int)(keys[i] & 0x7fffffffull);
    bool forced = page < sink || page >= first_diag;
    nf_local += !forced;
  }
  int nf_before = block_excl_scan(nf_local, warp_sums, nullptr);
  // mark selection into the low bit field's spare bit (bit 31 of the page field
  // is unused because pages < 2^31 - 1): reuse keys[] in place
  int sel_local = 0;
  for (int i = beg; i < beg + per && i < n_b; ++i) {
    int page = 0x7fffffff - (int)(keys[i] & 0x7fffffffull);
    bool forced = page < sink || page >= first_diag;
    bool sel = forced || (nf_before < quota);
    if (!forced) ++nf_before;
    sel_local += sel;
    keys[i] = sel ? (unsigned long long)page : ~0ull;  // page id or "dropped"
  }
  int total = 0;
  int out_before = block_excl_scan(sel_local, warp_sums, &total);
  int32_t* orow = order + row * k_cap;
  if (!ascending) {
    for (int i = beg; i < beg + per && i < n_b; ++i) {
      if (keys[i] != ~0ull) orow[out_before++] = (int32_t)keys[i];
    }
  } else {
    // list the kept pages by page id: flag array over pages, then compact
    __syncthreads();
    int* flag = reinterpret_cast<int*>(keys + npow2);  // second half of smem
    for (int p = threadIdx.x; p < n_b; p += blockDim.x) flag[p] = 0;
    __syncthreads();
    for (int i = beg; i < beg + per && i < n_b; ++i)
      if (keys[i] != ~0ull) flag[(int)keys[i]] = 1;
    __syncthreads();
    const int perp = (n_b + blockDim.x - 1) / blockDim.x;
    const int bp = threadIdx.x * perp;
    int cnt = 0;
    for (int p = bp; p < bp + perp && p < n_b; ++p) cnt += flag[p];
    int pos = block_excl_scan(cnt, warp_sums, nullptr);
    for (int p = bp; p < bp + perp && p < n_b; ++p)
      if (flag[p]) orow[pos++] = p;
  }
  for (int j = total + threadIdx.x; j < k_cap; j += blockDim.x) orow[j] = -1;
  if (threadIdx.x == 0) {
    count[row] = total;
    if (total != k_b) set_status(COSA_ERR_INVALID_ARG);  // cannot happen for valid shapes
  }
}

}  // namespace cosa
