// Kernel-Aware Proxy scores on the tensor cores (gist.science/pt "CoSA"
// technical summary, §2.2: "computa scores aproximados e aplica MaxPool sobre
// as chaves").
//
// For one (batch, KV head) slab the pooled queries of all q-blocks and all G
// heads of the group form the rows of A (row = (qb, g, r)) and the pooled keys
// form the rows of B (sub-key s = page * T + t); scores are scale * A B^T.
// Accuracy: the logits grow large with long contexts (hundreds), and the
// ranking needs them to fp32 precision, so each operand is split into two TF32
// terms (x = hi + lo, both TF32) and A B^T = hi hi + hi lo + lo hi up to a
// lo lo term of relative size 2^-22, with fp32 accumulation (kind::tf32).
//
// One CTA (192 threads) per tile of 128 rows of one slab, looping over
// 128-sub-key column tiles up to the causal limit of its last row:
//   warp 0     TMA: the A tile (hi and lo, resident), then B chunks of 32
//              fp32 (one 128-byte swizzle atom) through a 3-stage ring;
//   warp 1     MMA issuer: 3 tf32 MMAs per 8-wide K step into one of two
//              128-column TMEM accumulators;
//   warps 2-5  epilogue, thread = row = TMEM lane: MaxPool over each page's T
//              sub-keys with causal visibility (sub-key visible iff its first
//              token <= the representative's last row), page maxima a[row][p]
//              written to the triangular array, running row max and the first
//              page attaining it kept in registers and written at the end.
// Triangular layout: slab s, q-block qb, row (g, r):
//   a + s * GR * cum(nQB) + GR * cum(qb) + (g R + r) * n_b(qb) + p,  p < n_b(qb).
#pragma once

#include "common.cuh"
#include "kap.cuh"
#include "tc_ptx.cuh"

namespace cosa {

struct ScoreParams {
  float* a;
  float* row_max;
  int* row_arg;
  int group, R, T, num_q_blocks, q_block, page_size, q_sub, k_sub;
  int rows_per_slab;   // nQB * G * R
  int keys_per_slab;   // nP * T
  int tiles_per_slab;  // ceil(rows_per_slab / 128)
  float scale;
  unsigned long long timeout_ns;
};

template <int D>
struct ScoreCfg {
  static constexpr int BM = 128, BN = 128, KC = 32;       // rows, sub-keys, K chunk (fp32)
  static constexpr int NKC = D / KC;                      // K chunks per row
  static constexpr int STAGES = 3;
  static constexpr uint32_t CHUNK = BM * KC * 4;          // one [128][32 fp32] box, 16 KB
  static constexpr uint32_t OFF_A = 0;                    // [hi, lo][NKC] chunks, resident
  static constexpr uint32_t OFF_B = OFF_A + 2 * NKC * CHUNK;
  static constexpr uint32_t STAGE = 2 * CHUNK;            // B hi + lo of one K chunk
  static constexpr uint32_t OFF_BAR = OFF_B + STAGES * STAGE;
  // a_full, b_full[S], b_empty[S], acc_full[2], acc_empty[2], done
  static constexpr int NBAR = 1 + 2 * STAGES + 4 + 1;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t SMEM_ALLOC = OFF_MISC + 16 + 1024;
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
};

template <int D, int T>
__global__ void __launch_bounds__(192, 1)
    kap_score_tc(const __grid_constant__ CUtensorMap tm_qhi, const __grid_constant__ CUtensorMap tm_qlo,
                 const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
                 const ScoreParams prm) {
  using C = ScoreCfg<D>;
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const uint32_t sb0 = (sraw + 1023u) & ~1023u;
  uint8_t* sg = smem_raw + (sb0 - sraw);
  const uint32_t sA = sb0 + C::OFF_A, sB = sb0 + C::OFF_B, bar = sb0 + C::OFF_BAR;
  const uint32_t b_afull = bar;
  auto b_bfull = [&](int s) { return bar + 8u * (1 + s); };
  auto b_bempty = [&](int s) { return bar + 8u * (1 + C::STAGES + s); };
  auto b_accfull = [&](int s) { return bar + 8u * (1 + 2 * C::STAGES + s); };
  auto b_accempty = [&](int s) { return bar + 8u * (3 + 2 * C::STAGES + s); };
  const uint32_t b_done = bar + 8u * (C::NBAR - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sg + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + C::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (__syncthreads_or(*(volatile int*)&g_status == COSA_ERR_TIMEOUT)) return;

  // heaviest row tiles of a slab first; slabs in order (their pooled keys stay in L2)
  const int slab = blockIdx.x / prm.tiles_per_slab;
  const int tile = prm.tiles_per_slab - 1 - blockIdx.x % prm.tiles_per_slab;
  const int row0 = tile * C::BM;
  const int GR = prm.group * prm.R;
  const int last_row = min(row0 + C::BM, prm.rows_per_slab) - 1;
  const int ns_max = T * causal_pages(last_row / GR, prm.q_block, prm.page_size);
  const int ntile = (ns_max + C::BN - 1) / C::BN;
  const int grow0 = slab * prm.rows_per_slab + row0;       // A row in the 2-D map
  const int gkey0 = slab * prm.keys_per_slab;               // B row in the 2-D map

  if (tid == 0) {
    mbar_init(b_afull, 1);
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(b_bfull(s), 1); mbar_init(b_bempty(s), 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(b_accfull(s), 1); mbar_init(b_accempty(s), 4); }
    mbar_init(b_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(sb0 + C::OFF_MISC, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const unsigned long long tmo = prm.timeout_ns;
  auto wait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    if (mbar_try_wait(bar_addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t spins = 0;
    while (!mbar_try_wait_sleep(bar_addr, parity, 20000u)) {
      if (*abort_flag) return false;
      if ((++spins & 3u) == 0 &&
          (*(volatile int*)&g_status == COSA_ERR_TIMEOUT || globaltimer_ns() - t0 > tmo)) {
        *abort_flag = 1;
        set_status(COSA_ERR_TIMEOUT);
        return false;
      }
    }
    return true;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ================= TMA producer =================
      prefetch_tmap(&tm_qhi);
      prefetch_tmap(&tm_khi);
      mbar_arrive_expect_tx(b_afull, 2 * C::NKC * C::CHUNK);
#pragma unroll
      for (int kc = 0; kc < C::NKC; ++kc) {
        tma_load_2d(sA + kc * C::CHUNK, &tm_qhi, b_afull, kc * C::KC, grow0);
        tma_load_2d(sA + (C::NKC + kc) * C::CHUNK, &tm_qlo, b_afull, kc * C::KC, grow0);
      }
      int issued = 0;
      for (int ct = 0; ct < ntile; ++ct) {
        bool ok = true;
        for (int kc = 0; kc < C::NKC; ++kc) {
          const int it = ct * C::NKC + kc, s = it % C::STAGES;
          if (it >= C::STAGES && !wait(b_bempty(s), ((it / C::STAGES) - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(b_bfull(s), C::STAGE);
          tma_load_2d(sB + s * C::STAGE, &tm_khi, b_bfull(s), kc * C::KC, gkey0 + ct * C::BN);
          tma_load_2d(sB + s * C::STAGE + C::CHUNK, &tm_klo, b_bfull(s), kc * C::KC,
                      gkey0 + ct * C::BN);
          ++issued;
        }
        if (!ok) break;
      }
      if (*abort_flag) {  // drain what was issued and never consumed
        const uint64_t t0 = globaltimer_ns();
        drain_wait(b_afull, 0, t0, tmo);
        for (int it = max(0, issued - C::STAGES); it < issued; ++it)
          drain_wait(b_bfull(it % C::STAGES), (it / C::STAGES) & 1, t0, tmo);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================= MMA issuer =================
      constexpr uint32_t ID = idesc_tf32_f32(C::BM, C::BN);
      bool ok = wait(b_afull, 0);
      for (int ct = 0; ok && ct < ntile; ++ct) {
        const int buf = ct & 1;
        if (ct >= 2 && !wait(b_accempty(buf), ((ct >> 1) - 1) & 1)) break;
        const uint32_t acc = tmem + buf * C::BN;
        for (int kc = 0; kc < C::NKC; ++kc) {
          const int it = ct * C::NKC + kc, s = it % C::STAGES;
          if (!wait(b_bfull(s), (it / C::STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < C::KC / 8; ++ks) {
            const uint64_t ah = smem_desc_sw128(sA + kc * C::CHUNK + ks * 32, 16, 1024);
            const uint64_t al = smem_desc_sw128(sA + (C::NKC + kc) * C::CHUNK + ks * 32, 16, 1024);
            const uint64_t bh = smem_desc_sw128(sB + s * C::STAGE + ks * 32, 16, 1024);
            const uint64_t bl = smem_desc_sw128(sB + s * C::STAGE + C::CHUNK + ks * 32, 16, 1024);
            mma_tf32_ss(acc, ah, bh, ID, (kc > 0 || ks > 0) ? 1u : 0u);
            mma_tf32_ss(acc, ah, bl, ID, 1u);
            mma_tf32_ss(acc, al, bh, ID, 1u);
          }
          mma_commit(b_bempty(s));
        }
        if (!ok) break;
        mma_commit(b_accfull(buf));
      }
      mma_commit(b_done);
      const uint64_t t0 = globaltimer_ns();
      drain_wait(b_done, 0, t0, tmo);
    }
  } else {
    // ================= epilogue: thread = row = TMEM lane =================
    const int q4 = warp & 3;
    const int i = q4 * 32 + lane;
    const int grow = row0 + i;
    const bool valid = grow < prm.rows_per_slab;
    const int qb = valid ? grow / GR : 0, rr = valid ? grow % GR : 0, r = rr % prm.R;
    const int n_b = causal_pages(qb, prm.q_block, prm.page_size);
    const int rep_last = qb * prm.q_block + (r + 1) * prm.q_sub - 1;
    float* arow = prm.a + (long long)slab * GR * cum_pages(prm.num_q_blocks, prm.q_block, prm.page_size) +
                  (long long)GR * cum_pages(qb, prm.q_block, prm.page_size) + (long long)rr * n_b;
    const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
    const int P = prm.page_size, ksub = prm.k_sub;
    const float scale = prm.scale;
    float m = -INFINITY;
    int arg = 0x7fffffff;
    for (int ct = 0; ct < ntile; ++ct) {
      const int buf = ct & 1;
      if (!__all_sync(0xffffffffu, wait(b_accfull(buf), (ct >> 1) & 1))) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < C::BN / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(t_row + buf * C::BN + c * 32, raw);
        const int s0 = ct * C::BN + c * 32;  // sub-key of column 0 (a multiple of T)
        const int pg0 = s0 / T;
        constexpr int NPG = 32 / T;          // pages of this chunk
        float v[NPG];
#pragma unroll
        for (int k = 0; k < NPG; ++k) {
          const int pg = pg0 + k;
          v[k] = -INFINITY;
#pragma unroll
          for (int t = 0; t < T; ++t) {
            if (pg * P + t * ksub <= rep_last) v[k] = fmaxf(v[k], __uint_as_float(raw[k * T + t]) * scale);
          }
          if (valid && pg < n_b && v[k] > m) { m = v[k]; arg = pg; }
        }
        // the chunk's page maxima with the widest stores the row's alignment allows
        // (one row per thread: scalar stores send a request per page and row)
        if (valid && pg0 < n_b) {
          float* dst = arow + pg0;
          const uintptr_t ad = reinterpret_cast<uintptr_t>(dst);
          if (pg0 + NPG <= n_b && NPG % 4 == 0 && (ad & 15) == 0) {
#pragma unroll
            for (int k = 0; k < NPG; k += 4)
              *reinterpret_cast<float4*>(dst + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
          } else if (pg0 + NPG <= n_b && NPG % 2 == 0 && (ad & 7) == 0) {
#pragma unroll
            for (int k = 0; k < NPG; k += 2)
              *reinterpret_cast<float2*>(dst + k) = make_float2(v[k], v[k + 1]);
          } else {
#pragma unroll
            for (int k = 0; k < NPG; ++k)
              if (pg0 + k < n_b) dst[k] = v[k];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_accempty(buf));
    }
    if (valid) {
      prm.row_max[(long long)slab * prm.rows_per_slab + grow] = m;
      prm.row_arg[(long long)slab * prm.rows_per_slab + grow] = arg;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace cosa
