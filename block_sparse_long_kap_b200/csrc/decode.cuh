// Decode with ordered skipping: one new query per sequence and head visits an
// ordered list of KV pages under the in-kernel rule of gist.science/pt §2.3
// ("Saltado no Kernel": a page is skipped when its local max lies more than
// ln(1/eps) below the running max), as a q-block of one row.  The pages leave
// decoding as future work (closing section); this is the plainest continuation.
//
// A single row makes the work bandwidth-bound (every listed K page is read once,
// every kept V page once, 2*P*D flops per page), so the kernels use CUDA cores and
// coalesced 16-byte loads, and split each list over many CTAs:
//   decode_qk_kernel   one warp per listed page: the page's P logits (scale folded
//                      in, log2 units, keys past the query masked) into the
//                      workspace, and the page's local max
//   decode_pv_kernel   per chunk of the list: the decisions, then the kept pages'
//                      exp2(s - M) V and row sum against M, the list's final max;
//                      the chunk that finishes last for its head adds the chunks'
//                      partial sums to O / l, the LSE and the computed count
// For eps <= 1 a skipped page's local max lies below the running max, so the
// running max before list position j is the max of the local maxima of all pages
// listed before j: every decision is known from the local maxima alone, and M, the
// max over the list, is the final running max (the page attaining it is kept), so
// no partial sum ever needs rescaling.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace cosa {

struct DecodeParams {
  const __nv_bfloat16* q;       // [B][H_q][D]
  const __nv_bfloat16* k_pool;  // [phys][H_kv][P][D]
  const __nv_bfloat16* v_pool;
  const int32_t* page_table;    // [B][pages_per_seq]
  const int32_t* positions;     // [B]
  const int32_t* order;         // [B][H_q][k_cap]
  const int32_t* count;         // [B][H_q]
  __nv_bfloat16* out;           // [B][H_q][D]
  float* lse;                   // [B][H_q] or null
  int32_t* computed;            // [B][H_q] or null
  uint8_t* skip_log;            // [B][H_q][k_cap] or null
  float* logits;                // workspace [B H_q][k_cap][P]
  float* mloc;                  // workspace [B H_q][k_cap]
  float* part_o;                // workspace [B H_q][n_chunks][D]
  float* part_l;                // workspace [B H_q][n_chunks]
  int* part_n;                  // workspace [B H_q][n_chunks]
  int* arrived;                 // workspace [B H_q]: chunks of the head done (reset by the logits pass)
  int num_q_heads, num_kv_heads, group, seq_len, pages_per_seq, num_phys_pages, k_cap, n_chunks;
  float scale_log2, log2_eps;
};

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = DEC_THREADS / 32;
constexpr int DEC_CHUNK = 16;  // list entries per CTA

// list entry j of head bh: its logical page, or -1 past the count or out of range
// (a page past the query's own page is an invalid list: reported, not read)
__device__ __forceinline__ int dec_page(const DecodeParams& p, long long bh, int j, int n, int t,
                                        int P) {
  if (j >= n) return -1;
  const int pg = __ldg(p.order + bh * p.k_cap + j);
  if (pg < 0 || pg > t / P) {
    set_status(COSA_ERR_INVALID_ARG);
    return -1;
  }
  return pg;
}

template <int D, int P>
__global__ void __launch_bounds__(DEC_THREADS) decode_qk_kernel(const DecodeParams p) {
  constexpr int LPR = D / 8;     // lanes per key row (16 bytes each)
  constexpr int RPI = 32 / LPR;  // key rows per warp-wide load
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  const int b = (int)(bh / p.num_q_heads), h = (int)(bh % p.num_q_heads);
  const int hk = h / p.group;
  const int t = __ldg(p.positions + b);
  const bool t_ok = t >= 0 && t < p.seq_len;
  const int n = t_ok ? min(max(__ldg(p.count + bh), 0), p.k_cap) : 0;
  if (blockIdx.x == 0) {
    // the P V pass counts this head's chunks in; a head with nothing to visit (an
    // empty list, or a position out of range: reported) gets its outputs here
    if (threadIdx.x == 0) {
      p.arrived[bh] = 0;
      if (!t_ok) set_status(COSA_ERR_INVALID_ARG);
      if (n == 0) {
        if (p.lse) p.lse[bh] = -INFINITY;
        if (p.computed) p.computed[bh] = 0;
      }
    }
    if (n == 0)
      for (int d = threadIdx.x; d < D; d += DEC_THREADS) p.out[bh * D + d] = __float2bfloat16_rn(0.f);
  }
  if (n == 0) return;
  // this lane's 8 query dims (scale and log2 e folded in)
  float qv[8];
  {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.q + bh * D) + (lane % LPR));
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h2[i]);
      qv[2 * i] = f.x * p.scale_log2;
      qv[2 * i + 1] = f.y * p.scale_log2;
    }
  }
  for (int jj = warp; jj < DEC_CHUNK; jj += DEC_WARPS) {
    const int j = blockIdx.x * DEC_CHUNK + jj;
    const int pg = dec_page(p, bh, j, n, t, P);
    if (pg < 0) {
      if (j < n && lane == 0) p.mloc[bh * p.k_cap + j] = -INFINITY;  // invalid entry: not read
      continue;
    }
    const int phys = __ldg(p.page_table + (long long)b * p.pages_per_seq + pg);
    if (phys < 0 || phys >= p.num_phys_pages) {  // outside the pool: reported, not read
      if (lane == 0) {
        set_status(COSA_ERR_INVALID_ARG);
        p.mloc[bh * p.k_cap + j] = -INFINITY;
      }
      continue;
    }
    const uint4* kp = reinterpret_cast<const uint4*>(
        p.k_pool + ((long long)phys * p.num_kv_heads + hk) * P * D);
    float* lrow = p.logits + (bh * p.k_cap + j) * P;
    float mx = -INFINITY;
    constexpr int IT = P / RPI;  // warp-wide loads per page
    constexpr int UN = 8;        // loads in flight
#pragma unroll 1
    for (int i0 = 0; i0 < IT; i0 += UN) {
      uint4 raw[UN];
#pragma unroll
      for (int u = 0; u < UN; ++u) raw[u] = __ldg(kp + (i0 + u) * 32 + lane);
#pragma unroll
      for (int u = 0; u < UN; ++u) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          acc = fmaf(qv[2 * e], f.x, acc);
          acc = fmaf(qv[2 * e + 1], f.y, acc);
        }
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        const int key = (i0 + u) * RPI + lane / LPR;  // key within the page
        const float s = (pg * P + key <= t) ? acc : -INFINITY;
        mx = fmaxf(mx, s);
        if (lane % LPR == 0) lrow[key] = s;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) p.mloc[bh * p.k_cap + j] = mx;
  }
}

template <int D, int P>
__global__ void __launch_bounds__(DEC_THREADS) decode_pv_kernel(const DecodeParams p) {
  constexpr int LPR = D / 8;
  constexpr int RPI = 32 / LPR;
  __shared__ float red_m[DEC_WARPS][2];
  __shared__ float o_s[DEC_WARPS][D];
  __shared__ float l_s[DEC_WARPS];
  __shared__ int keep_s[DEC_CHUNK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  const int b = (int)(bh / p.num_q_heads), h = (int)(bh % p.num_q_heads);
  const int hk = h / p.group;
  const int t = __ldg(p.positions + b);
  if (t < 0 || t >= p.seq_len) return;
  const int n = min(max(__ldg(p.count + bh), 0), p.k_cap);
  const int j0 = blockIdx.x * DEC_CHUNK;
  if (j0 >= n) return;
  const float* ml = p.mloc + bh * p.k_cap;
  // the max over the list before this chunk, and over the whole list
  float mb = -INFINITY, ma = -INFINITY;
  for (int j = threadIdx.x; j < n; j += DEC_THREADS) {
    const float v = ml[j];
    ma = fmaxf(ma, v);
    if (j < j0) mb = fmaxf(mb, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, o));
  }
  if (lane == 0) { red_m[warp][0] = mb; red_m[warp][1] = ma; }
  __syncthreads();
  mb = red_m[0][0];
  ma = red_m[0][1];
#pragma unroll
  for (int w = 1; w < DEC_WARPS; ++w) { mb = fmaxf(mb, red_m[w][0]); ma = fmaxf(ma, red_m[w][1]); }
  // decisions of this chunk: page j is skipped iff j >= 1 and its local max lies
  // below ln(eps) of the max of the local maxima listed before it
  if (warp == 0) {
    const int j = j0 + lane;
    const float v = (lane < DEC_CHUNK && j < n) ? ml[j] : -INFINITY;
    float inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc = fmaxf(inc, y);
    }
    float before = __shfl_up_sync(0xffffffffu, inc, 1);
    before = fmaxf(mb, lane == 0 ? -INFINITY : before);
    if (lane < DEC_CHUNK && j < n) {
      const bool keep = j == 0 || !(v - before < p.log2_eps);
      keep_s[lane] = keep ? 1 : 0;
      if (p.skip_log) p.skip_log[bh * p.k_cap + j] = keep ? 0 : 1;
    } else if (lane < DEC_CHUNK) {
      keep_s[lane] = 0;
    }
  }
  __syncthreads();
  // P V over the chunk's kept pages: lane l accumulates dims (l % LPR) * 8 .. + 8 of
  // the rows l / LPR (mod RPI)
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float lsum = 0.f;
  for (int jj = warp; jj < DEC_CHUNK; jj += DEC_WARPS) {
    const int j = j0 + jj;
    if (j >= n || !keep_s[jj]) continue;
    const int pg = __ldg(p.order + bh * p.k_cap + j);
    if (pg < 0 || pg > t / P) continue;  // an invalid entry (reported by the logits pass)
    const int phys = __ldg(p.page_table + (long long)b * p.pages_per_seq + pg);
    if (phys < 0 || phys >= p.num_phys_pages) continue;  // reported by the logits pass
    const uint4* vp = reinterpret_cast<const uint4*>(
        p.v_pool + ((long long)phys * p.num_kv_heads + hk) * P * D);
    const float* lrow = p.logits + (bh * p.k_cap + j) * P;
    constexpr int IT = P / RPI;
    constexpr int UN = 8;
#pragma unroll 1
    for (int i0 = 0; i0 < IT; i0 += UN) {
      uint4 raw[UN];
#pragma unroll
      for (int u = 0; u < UN; ++u) raw[u] = __ldg(vp + (i0 + u) * 32 + lane);
#pragma unroll
      for (int u = 0; u < UN; ++u) {
        const int key = (i0 + u) * RPI + lane / LPR;
        const float s = lrow[key];
        const float w = s == -INFINITY ? 0.f : tc::ex2_approx(s - ma);
        if (lane % LPR == 0) lsum += w;
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
        }
      }
    }
  }
  // lanes holding the same dims (l, l + LPR, ...) are summed; then the warps
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  if (lane < LPR)
#pragma unroll
    for (int e = 0; e < 8; ++e) o_s[warp][lane * 8 + e] = acc[e];
  if (lane == 0) l_s[warp] = lsum;
  __syncthreads();
  const long long pc = bh * p.n_chunks + blockIdx.x;
  for (int d = threadIdx.x; d < D; d += DEC_THREADS) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < DEC_WARPS; ++w) v += o_s[w][d];
    p.part_o[pc * D + d] = v;
  }
  __shared__ int last_s;
  if (threadIdx.x == 0) {
    float l = 0.f;
    int kept = 0;
#pragma unroll
    for (int w = 0; w < DEC_WARPS; ++w) l += l_s[w];
    for (int jj = 0; jj < DEC_CHUNK; ++jj) kept += keep_s[jj];
    p.part_l[pc] = l;
    p.part_n[pc] = kept;
  }
  // the chunk that finishes last for this head combines (every chunk's partial sums
  // are made visible before it counts itself in)
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int nc = (n + DEC_CHUNK - 1) / DEC_CHUNK;
    last_s = atomicAdd(p.arrived + bh, 1) == nc - 1;
    if (last_s) __threadfence();
  }
  __syncthreads();
  if (!last_s) return;
  const int nc = (n + DEC_CHUNK - 1) / DEC_CHUNK;
  const long long pc0 = bh * p.n_chunks;
  __shared__ float l_tot;
  if (threadIdx.x == 0) {
    float l = 0.f;
    int kept = 0;
    for (int c = 0; c < nc; ++c) {
      l += ((volatile float*)p.part_l)[pc0 + c];
      kept += ((volatile int*)p.part_n)[pc0 + c];
    }
    l_tot = l;
    if (p.computed) p.computed[bh] = kept;
    if (p.lse) p.lse[bh] = l > 0.f ? (ma + log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
  __syncthreads();
  const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
  for (int d = threadIdx.x; d < D; d += DEC_THREADS) {
    float o = 0.f;
    for (int c = 0; c < nc; ++c) o += ((volatile float*)p.part_o)[(pc0 + c) * D + d];
    p.out[bh * D + d] = __float2bfloat16_rn(o * inv);
  }
}

}  // namespace cosa
