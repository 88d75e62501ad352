// Ordered-Skipping Kernel and dense causal attention, warp-level MMA version.
// (gist.science/pt "CoSA" technical summary, §2.3 "Estágio 2: OSK".)
//
// One CTA per (b, h_q, q-block) tile of BQ rows; BQ/16 warps, 16 rows each.
// The CTA walks the q-block's page list in list order; each page's K and V
// tiles are fetched through the page table ("Saltado pela Máscara": pages not
// in the list are never read) into a two-stage cp.async ring.  After QK^T the
// warps vote: a page other than the first is skipped when no row of the tile
// has (page max - running max) >= log2(eps) in the log2 domain ("Saltado no
// Kernel"); otherwise online softmax and PV run ("Computado").
#pragma once

#include "common.cuh"

namespace cosa {

struct AttnParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_pool;
  const __nv_bfloat16* v_pool;
  const int32_t* page_table;
  const int32_t* order;   // null for dense
  const int32_t* count;   // null for dense
  __nv_bfloat16* out;
  float* lse;             // optional
  int32_t* computed;      // optional
  uint8_t* skip_log;      // optional
  int num_q_heads, num_kv_heads, group, seq_len, num_q_blocks, pages_per_seq, k_cap;
  float scale_log2;       // softmax_scale * log2(e)
  float log2_eps;         // log2(eps); -inf disables skipping
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Row-major [rows][D] bf16 tile with 16-byte chunks XOR-swizzled by row.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  return (uint32_t)((row * CPR + (chunk ^ (row & 7))) * 16);
}

template <int D>
__device__ __forceinline__ void load_tile_async(uint32_t sbase, const __nv_bfloat16* g, int rows,
                                                int tid, int nthreads) {
  constexpr int CPR = D / 8;
  for (int i = tid; i < rows * CPR; i += nthreads) {
    int r = i / CPR, c = i % CPR;
    cp_async16(sbase + swz<D>(r, c), g + (long long)r * D + c * 8);
  }
}

template <int D, int P, int BQ, bool DENSE>
__global__ void __launch_bounds__(BQ * 2) attn_mma_kernel(AttnParams prm) {
  constexpr int NW = BQ / 16;
  constexpr int NT = NW * 32;
  constexpr int KS = D / 16;   // k-steps for QK^T
  constexpr int NTS = P / 8;   // n-tiles of S
  constexpr int NTO = D / 8;   // n-tiles of O
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* Ks = Qs + BQ * D;          // [2][P][D]
  __nv_bfloat16* Vs = Ks + 2 * P * D;       // [2][P][D]
  __shared__ int votes[2][NW];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;

  // work decode: KV-head major so that concurrently running CTAs share K/V in L2
  const int G = prm.group;
  const int per_kv = G * prm.num_q_blocks;
  const int z = blockIdx.x / per_kv;
  const int rem = blockIdx.x % per_kv;
  const int qb = prm.num_q_blocks - 1 - rem / G;
  const int hk = z % prm.num_kv_heads;
  const int b = z / prm.num_kv_heads;
  const int h = hk * G + rem % G;
  const long long bh = (long long)b * prm.num_q_heads + h;
  const int row0 = qb * BQ;

  const int n_causal = causal_pages(qb, BQ, P);
  int n_list = n_causal;
  const int32_t* olist = nullptr;
  if (!DENSE) {
    olist = prm.order + (bh * prm.num_q_blocks + qb) * prm.k_cap;
    n_list = min(max(prm.count[bh * prm.num_q_blocks + qb], 0), prm.k_cap);
    // every listed page must be a causal page of this q-block; otherwise flag
    // the call and produce no output for the tile
    int bad = 0;
    for (int j = tid; j < n_list; j += NT) bad |= (olist[j] < 0) | (olist[j] >= n_causal);
    if (__syncthreads_or(bad)) {
      if (tid == 0) set_status(COSA_ERR_INVALID_ARG);
      n_list = 0;
    }
  }
  const int32_t* ptab = prm.page_table + (long long)b * prm.pages_per_seq;

  const uint32_t sQ = smem_u32(Qs), sK = smem_u32(Ks), sV = smem_u32(Vs);
  load_tile_async<D>(sQ, prm.q + (bh * prm.seq_len + row0) * D, BQ, tid, NT);
  cp_async_commit();
  auto issue_page = [&](int j) {
    int page = DENSE ? j : olist[j];
    long long phys = ptab[page];
    long long off = (phys * prm.num_kv_heads + hk) * (long long)P * D;
    int st = j & 1;
    load_tile_async<D>(sK + st * P * D * 2, prm.k_pool + off, P, tid, NT);
    load_tile_async<D>(sV + st * P * D * 2, prm.v_pool + off, P, tid, NT);
    cp_async_commit();
  };
  if (n_list > 0) {
    issue_page(0);
    cp_async_wait<1>();
  } else {
    cp_async_wait<0>();
  }
  __syncthreads();

  // Q fragments for this warp's 16 rows
  uint32_t qf[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
    int c = 2 * ks + (lane >> 4);
    ldsm_x4(sQ + swz<D>(r, c), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
  }

  float o[NTO][4];
#pragma unroll
  for (int i = 0; i < NTO; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  const int rowA = row0 + warp * 16 + g, rowB = rowA + 8;
  int n_computed = 0;

  for (int j = 0; j < n_list; ++j) {
    if (j + 1 < n_list) {
      issue_page(j + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int st = j & 1;
    const int page = DENSE ? j : olist[j];
    const uint32_t kb = sK + st * P * D * 2, vb = sV + st * P * D * 2;

    float s[NTS][4];
#pragma unroll
    for (int i = 0; i < NTS; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int np = 0; np < NTS / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        int r = np * 16 + (lane & 7) + (lane >> 4) * 8;
        int c = 2 * ks + ((lane >> 3) & 1);
        ldsm_x4(kb + swz<D>(r, c), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[ks], b0, b1);
        mma_bf16(s[2 * np + 1], qf[ks], b2, b3);
      }
    }
    // scale into the log2 domain, causal mask on pages reaching past the first row
    const int key0 = page * P;
    const bool diag = key0 + P - 1 > row0;
    float mloc[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < NTS; ++i) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[i][e] * prm.scale_log2;
        if (diag) {
          int key = key0 + i * 8 + 2 * t4 + (e & 1);
          int row = (e < 2) ? rowA : rowB;
          if (key > row) v = -INFINITY;
        }
        s[i][e] = v;
        mloc[e >> 1] = fmaxf(mloc[e >> 1], v);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mloc[r] = fmaxf(mloc[r], __shfl_xor_sync(0xffffffffu, mloc[r], 1));
      mloc[r] = fmaxf(mloc[r], __shfl_xor_sync(0xffffffffu, mloc[r], 2));
    }
    bool skip = false;
    if (!DENSE && j > 0) {
      bool need = false;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        bool live = mloc[r] != -INFINITY;
        need |= live && (m_run[r] == -INFINITY || (mloc[r] - m_run[r]) >= prm.log2_eps);
      }
      need = __any_sync(0xffffffffu, need);
      if (lane == 0) votes[j & 1][warp] = need ? 1 : 0;
      __syncthreads();
      bool any = false;
#pragma unroll
      for (int w = 0; w < NW; ++w) any |= votes[j & 1][w] != 0;
      skip = !any;
    }
    if (!DENSE && tid == 0 && prm.skip_log)
      prm.skip_log[(bh * prm.num_q_blocks + qb) * prm.k_cap + j] = skip ? 1 : 0;
    if (!skip) {
      ++n_computed;
      float alpha[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float mn = fmaxf(m_run[r], mloc[r]);
        float mu = (mn == -INFINITY) ? 0.f : mn;
        alpha[r] = exp2f(m_run[r] - mu);
        m_run[r] = mn;
        mloc[r] = mu;  // reuse as the exponent base
      }
      float rs[2] = {0.f, 0.f};
      uint32_t pf[NTS / 2][4];
#pragma unroll
      for (int i = 0; i < NTS; ++i) {
        float p0 = exp2f(s[i][0] - mloc[0]);
        float p1 = exp2f(s[i][1] - mloc[0]);
        float p2 = exp2f(s[i][2] - mloc[1]);
        float p3 = exp2f(s[i][3] - mloc[1]);
        rs[0] += p0 + p1;
        rs[1] += p2 + p3;
        pf[i >> 1][(i & 1) * 2 + 0] = pack_bf16(p0, p1);
        pf[i >> 1][(i & 1) * 2 + 1] = pack_bf16(p2, p3);
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 1);
        rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 2);
        l_run[r] = l_run[r] * alpha[r] + rs[r];
      }
#pragma unroll
      for (int i = 0; i < NTO; ++i) {
        o[i][0] *= alpha[0];
        o[i][1] *= alpha[0];
        o[i][2] *= alpha[1];
        o[i][3] *= alpha[1];
      }
      // PV: A = P (k = keys), B = V [key][d] via transposed ldmatrix
#pragma unroll
      for (int kk = 0; kk < P / 16; ++kk) {
        uint32_t a[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
#pragma unroll
        for (int dn = 0; dn < NTO / 2; ++dn) {
          uint32_t b0, b1, b2, b3;
          int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          int c = 2 * dn + (lane >> 4);
          ldsm_x4_t(vb + swz<D>(r, c), b0, b1, b2, b3);
          mma_bf16(o[2 * dn], a, b0, b1);
          mma_bf16(o[2 * dn + 1], a, b2, b3);
        }
      }
    }
    __syncthreads();
  }

  // epilogue
  float inv[2], lse2[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    inv[r] = l_run[r] > 0.f ? 1.f / l_run[r] : 0.f;
    lse2[r] = l_run[r] > 0.f ? (m_run[r] + log2f(l_run[r])) * 0.69314718055994531f : -INFINITY;
  }
  __nv_bfloat16* orow = prm.out + (bh * prm.seq_len + row0 + warp * 16) * D;
#pragma unroll
  for (int i = 0; i < NTO; ++i) {
    int col = i * 8 + 2 * t4;
    *reinterpret_cast<uint32_t*>(orow + g * D + col) = pack_bf16(o[i][0] * inv[0], o[i][1] * inv[0]);
    *reinterpret_cast<uint32_t*>(orow + (g + 8) * D + col) =
        pack_bf16(o[i][2] * inv[1], o[i][3] * inv[1]);
  }
  if (prm.lse && t4 == 0) {
    prm.lse[bh * prm.seq_len + rowA] = lse2[0];
    prm.lse[bh * prm.seq_len + rowB] = lse2[1];
  }
  if (!DENSE && prm.computed && tid == 0)
    prm.computed[bh * prm.num_q_blocks + qb] = n_computed;
}

}  // namespace cosa
