// Ordered-Skipping Kernel (and dense causal attention) on the sm_100a tensor
// cores: TMA page loads through the page table, tcgen05.mma into TMEM, one
// query row per TMEM lane.  (gist.science/pt "CoSA" technical summary,
// §2.3 "Estágio 2: OSK": mask-skipped pages are never loaded, "KV page
// remapping"; in-kernel skip from the page's local max vs the running max;
// computed pages get the full softmax + PV.)
//
// One CTA (384 threads) per (b, h_q, q-block) tile of up to 128 query rows:
//   warp 0      TMA producer: the Q tile once, then K of every listed page, in
//               list order, into a KS-stage ring (page table gives the
//               physical page; no multicast).
//   warp 1      QK^T issuer (one thread): S_j = Q K_j^T into one of SB TMEM
//               buffers, in list order.
//   warp 2      TMA producer for V: loads V_j only for pages the vote keeps,
//               so a skipped page costs its K tile and one QK^T, nothing more.
//   warp 3      PV issuer (one thread): for each kept page, once its P and V
//               tiles are ready, O += P_j V_j into the TMEM accumulator.  With
//               two issuing threads a late V never stalls QK^T.
//   warps 4-11  softmax, two warpgroups: warpgroup h (0/1) owns columns
//               [h P/2, (h+1) P/2) of every S tile and [h D/2, (h+1) D/2) of O;
//               thread (warp % 4, lane) owns query row 32 (warp % 4) + lane,
//               which is its TMEM lane.  Per page: read the half row of S,
//               mask the causal diagonal, take the half-row max, then one
//               barrier round among the 256 softmax threads exchanges the
//               half maxima and the votes.  The skip rule "some row has
//               (page max - running max) >= log2 eps" is decided exactly on
//               half rows, because max(a, b) - m >= t  <=>  a - m >= t or
//               b - m >= t.  The first listed page is always kept.  For kept
//               pages each thread writes P = exp2(s - m_ref) (bf16) for its
//               half row into a swizzled shared-memory tile; m_ref, the
//               exponent base, moves only when the running max passes it by
//               more than 2^8 (O and l are then rescaled in TMEM), which keeps
//               the result exact.
// Decisions reach the V producer and the PV issuer as sequence-tagged words in
// a shared-memory ring; their progress counters give the ring back-pressure.
// Every wait is bounded: on timeout the CTA records COSA_ERR_TIMEOUT in the
// status word, drains what it issued, frees TMEM and exits; a timed-out CTA
// makes every later CTA of the launch exit at once.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace cosa {

struct TcParams {
  const int32_t* page_table;
  const int32_t* order;   // null for dense
  const int32_t* count;   // null for dense
  __nv_bfloat16* out;
  float* lse;
  int32_t* computed;
  uint8_t* skip_log;
  int num_q_heads, num_kv_heads, group, seq_len, num_q_blocks, pages_per_seq, k_cap, q_block;
  float scale_log2, log2_eps;
  unsigned long long timeout_ns;
};

template <int D, int P>
struct TcCfg {
  static constexpr int QB = 128;                  // MMA M (rows per tile, padded)
  static constexpr int NT = 384;                  // 4 role warps + 2 softmax warpgroups
  static constexpr int HP = P / 2;                // S columns per softmax thread
  static constexpr int HD = D / 2;                // O columns per softmax thread
  static constexpr int KS = (P == 64) ? 6 : 2;    // K ring stages
  static constexpr int VS = 2;                    // V ring stages
  static constexpr int PS = (P == 64) ? 2 : 1;    // P tile ring stages
  static constexpr int SB = (P == 64) ? 4 : 3;    // S buffers in TMEM
  static constexpr int DS = 64;                   // decision ring (words)
  static constexpr uint32_t Q_BYTES = QB * D * 2;
  static constexpr uint32_t KV_BYTES = P * D * 2;
  static constexpr uint32_t P_BYTES = QB * P * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KS * KV_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + VS * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + PS * P_BYTES;
  // q, k_full/empty, v_full/empty, s_full/free, p_full/empty, done (QK), done (PV)
  static constexpr int NBAR = 1 + 2 * KS + 2 * VS + 2 * SB + 2 * PS + 2;
  static constexpr uint32_t OFF_MISC = (OFF_BAR + NBAR * 8 + 127) & ~127u;  // vector-aligned
  // misc: +0 TMEM address, +4 abort flag, +8 PV progress, +12 V progress,
  //       +16 votes [2 rounds][2 parities][8], +256 decision words [DS],
  //       +512 half-row maxima [2 parities][2 pages][2 halves][128],
  //       +4608 half-row sums [2][128]
  static constexpr uint32_t MISC_BYTES = 5632;
  static constexpr uint32_t SMEM = OFF_MISC + MISC_BYTES;
  static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;  // 1024-byte alignment slack
  static constexpr int COL_O = SB * P;
  static constexpr int TMEM_COLS = (SB * P + D <= 256) ? 256 : 512;
  static_assert(SB * P + D <= 512, "TMEM budget");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(256 + 4 * DS <= 512, "decision ring fits its slot");
  static_assert(OFF_MISC % 128 == 0, "16-byte vector access to the vote words");
};

constexpr float kRescaleLog2 = 8.0f;  // m_ref trails the running max by < 2^8

template <int D, int P, bool DENSE>
__global__ void __launch_bounds__(384, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const TcParams prm) {
  using C = TcCfg<D, P>;
  using namespace tc;
  constexpr int HP = C::HP, HD = C::HD;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const uint32_t sb0 = (sraw + 1023u) & ~1023u;
  uint8_t* sg = smem_raw + (sb0 - sraw);
  const uint32_t sQ = sb0 + C::OFF_Q, sK = sb0 + C::OFF_K, sV = sb0 + C::OFF_V,
                 sP = sb0 + C::OFF_P;
  const uint32_t bar = sb0 + C::OFF_BAR;
  const uint32_t b_q = bar;
  auto b_kfull = [&](int s) { return bar + 8u * (1 + s); };
  auto b_kempty = [&](int s) { return bar + 8u * (1 + C::KS + s); };
  auto b_vfull = [&](int s) { return bar + 8u * (1 + 2 * C::KS + s); };
  auto b_vempty = [&](int s) { return bar + 8u * (1 + 2 * C::KS + C::VS + s); };
  auto b_sfull = [&](int s) { return bar + 8u * (1 + 2 * C::KS + 2 * C::VS + s); };
  auto b_sfree = [&](int s) { return bar + 8u * (1 + 2 * C::KS + 2 * C::VS + C::SB + s); };
  auto b_pfull = [&](int s) { return bar + 8u * (1 + 2 * C::KS + 2 * C::VS + 2 * C::SB + s); };
  auto b_pempty = [&](int s) {
    return bar + 8u * (1 + 2 * C::KS + 2 * C::VS + 2 * C::SB + C::PS + s);
  };
  const uint32_t b_done_s = bar + 8u * (C::NBAR - 2);
  const uint32_t b_done_pv = bar + 8u * (C::NBAR - 1);
  uint8_t* misc = sg + C::OFF_MISC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* pv_pos = reinterpret_cast<volatile int*>(misc + 8);
  volatile int* v_pos = reinterpret_cast<volatile int*>(misc + 12);
  volatile int* votes = reinterpret_cast<volatile int*>(misc + 16);               // [2][2][8]
  volatile uint32_t* dec_word = reinterpret_cast<volatile uint32_t*>(misc + 256);  // [DS]
  volatile float* hmax = reinterpret_cast<volatile float*>(misc + 512);     // [2][2][2][128]
  volatile float* hsum = reinterpret_cast<volatile float*>(misc + 4608);    // [2][128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // a CTA that ran out of time anywhere in this launch stops the others early
  if (__syncthreads_or(*(volatile int*)&g_status == COSA_ERR_TIMEOUT)) return;

  // ---- work decode: KV-head major, heaviest q-blocks first, G heads fastest
  const int G = prm.group;
  const int per_kv = G * prm.num_q_blocks;
  const int z = blockIdx.x / per_kv;
  const int rem = blockIdx.x % per_kv;
  const int qb = prm.num_q_blocks - 1 - rem / G;
  const int hk = z % prm.num_kv_heads;
  const int b = z / prm.num_kv_heads;
  const int h = hk * G + rem % G;
  const long long bh = (long long)b * prm.num_q_heads + h;
  const int row0 = qb * prm.q_block;
  const int n_causal = causal_pages(qb, prm.q_block, P);
  int n_list = n_causal;
  const int32_t* olist = nullptr;
  if (!DENSE) {
    olist = prm.order + (bh * prm.num_q_blocks + qb) * prm.k_cap;
    n_list = min(max(prm.count[bh * prm.num_q_blocks + qb], 0), prm.k_cap);
    int bad = 0;
    for (int j = tid; j < n_list; j += blockDim.x) bad |= (olist[j] < 0) | (olist[j] >= n_causal);
    if (__syncthreads_or(bad)) {
      if (tid == 0) set_status(COSA_ERR_INVALID_ARG);
      n_list = 0;
    }
  }
  const int32_t* ptab = prm.page_table + (long long)b * prm.pages_per_seq;
  auto page_at = [&](int j) { return DENSE ? j : __ldg(olist + j); };

  // ---- setup
  if (tid == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < C::KS; ++s) { mbar_init(b_kfull(s), 1); mbar_init(b_kempty(s), 1); }
    for (int s = 0; s < C::VS; ++s) { mbar_init(b_vfull(s), 1); mbar_init(b_vempty(s), 1); }
    for (int s = 0; s < C::SB; ++s) { mbar_init(b_sfull(s), 1); mbar_init(b_sfree(s), 8); }
    for (int s = 0; s < C::PS; ++s) { mbar_init(b_pfull(s), 8); mbar_init(b_pempty(s), 1); }
    mbar_init(b_done_s, 1);
    mbar_init(b_done_pv, 1);
    *abort_flag = 0;
    *pv_pos = 0;
    *v_pos = 0;
    for (int s = 0; s < C::DS; ++s) dec_word[s] = 0xFFFFFFFFu;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(sb0 + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (prm.q_block < C::QB && warp >= 4) {
    // rows past the q-block are padding: zero them once (the TMA box fills the rest)
    const int pad = C::QB - prm.q_block;
    for (int i = tid - 128; i < pad * (D / 64) * 8; i += 256) {
      const int chunk = i & 7, r = prm.q_block + (i >> 3) % pad, kb = (i >> 3) / pad;
      st_shared_v4(sQ + kb * (C::QB * 128) + r * 128 + chunk * 16, 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const unsigned long long tmo = prm.timeout_ns;
  auto give_up = [&]() {
    *abort_flag = 1;
    set_status(COSA_ERR_TIMEOUT);
  };
  // bounded blocking wait on an mbarrier phase; false on timeout or abort
  auto wait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    if (mbar_try_wait(bar_addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t spins = 0;
    while (!mbar_try_wait_sleep(bar_addr, parity, 20000u)) {
      if (*abort_flag) return false;
      if ((++spins & 3u) == 0 &&
          (*(volatile int*)&g_status == COSA_ERR_TIMEOUT || globaltimer_ns() - t0 > tmo)) {
        give_up();
        return false;
      }
    }
    return true;
  };
  // bounded wait for the decision on page i; returns -1 on timeout, else 0/1
  auto decision = [&](int i) -> int {
    const uint32_t want = (uint32_t)i << 1;
    uint32_t w = dec_word[i % C::DS];
    if ((w & ~1u) == want) return (int)(w & 1u);
    const uint64_t t0 = globaltimer_ns();
    uint32_t spins = 0;
    while (((w = dec_word[i % C::DS]) & ~1u) != want) {
      if (*abort_flag) return -1;
      if ((++spins & 63u) == 0 &&
          (*(volatile int*)&g_status == COSA_ERR_TIMEOUT || globaltimer_ns() - t0 > tmo)) {
        give_up();
        return -1;
      }
      __nanosleep(64);  // leave the issue slots to the softmax warps sharing this scheduler
    }
    return (int)(w & 1u);
  };

  if (warp == 0) {
    // ================= Q / K producer (lane 0 issues; the warp prefetches page ids)
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      mbar_arrive_expect_tx(b_q, (uint32_t)((D / 64) * prm.q_block * 128));
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_3d(sQ + kb * (C::QB * 128), &tm_q, b_q, kb * 64, row0, (int)bh);
    }
    int issued = 0;
    bool ok = true;
    for (int base = 0; ok && base < n_list; base += 32) {
      const int jl = base + lane;
      const int cz_l = jl < n_list ? ptab[page_at(jl)] * prm.num_kv_heads + hk : 0;
      const int nb = min(32, n_list - base);
      for (int jj = 0; jj < nb; ++jj) {
        const int j = base + jj;
        const int cz = __shfl_sync(0xffffffffu, cz_l, jj);
        const int s = j % C::KS;
        if (j >= C::KS) {
          ok = __all_sync(0xffffffffu, wait(b_kempty(s), ((j / C::KS) - 1) & 1));
          if (!ok) break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(b_kfull(s), C::KV_BYTES);
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_3d(sK + s * C::KV_BYTES + kb * (P * 128), &tm_k, b_kfull(s), kb * 64, 0, cz);
        }
        ++issued;
        __syncwarp();
      }
    }
    if (lane == 0 && *abort_flag) {  // drain what was issued and never consumed
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(b_q, 0) && globaltimer_ns() - t0 < tmo) {}
      for (int j = max(0, issued - C::KS); j < issued; ++j)
        while (!mbar_try_wait(b_kfull(j % C::KS), (j / C::KS) & 1) &&
               globaltimer_ns() - t0 < tmo) {}
    }
  } else if (warp == 2) {
    // ================= V producer: only pages the vote keeps =================
    if (lane == 0) prefetch_tmap(&tm_v);
    int vc = 0;
    bool ok = true;
    for (int base = 0; ok && base < n_list; base += 32) {
      const int il = base + lane;
      const int cz_l = il < n_list ? ptab[page_at(il)] * prm.num_kv_heads + hk : 0;
      const int nb = min(32, n_list - base);
      for (int ii = 0; ii < nb; ++ii) {
        const int i = base + ii;
        const int cz = __shfl_sync(0xffffffffu, cz_l, ii);
        if (!DENSE && i > 0) {  // page 0 is always kept: its V goes out before the vote
          const int d = decision(i);
          ok = __all_sync(0xffffffffu, d >= 0);
          if (!ok) break;
          if (lane == 0) *v_pos = i + 1;
          if (d == 0) continue;
        }
        const int s = vc % C::VS;
        if (vc >= C::VS) {
          ok = __all_sync(0xffffffffu, wait(b_vempty(s), ((vc / C::VS) - 1) & 1));
          if (!ok) break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(b_vfull(s), C::KV_BYTES);
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_3d(sV + s * C::KV_BYTES + kb * (P * 128), &tm_v, b_vfull(s), kb * 64, 0, cz);
        }
        ++vc;
        __syncwarp();
        if (!DENSE && i == 0) {
          ok = __all_sync(0xffffffffu, decision(0) >= 0);
          if (!ok) break;
          if (lane == 0) *v_pos = 1;
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      const uint64_t t0 = globaltimer_ns();
      for (int c = max(0, vc - C::VS); c < vc; ++c)
        while (!mbar_try_wait(b_vfull(c % C::VS), (c / C::VS) & 1) &&
               globaltimer_ns() - t0 < tmo) {}
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================= QK^T issuer, list order =================
      constexpr uint32_t ID_QK = idesc_bf16_f32(128, P, 0);
      bool ok = wait(b_q, 0);
      for (int j = 0; ok && j < n_list; ++j) {
        const int ks = j % C::KS, sbuf = j % C::SB;
        if (!wait(b_kfull(ks), (j / C::KS) & 1)) break;
        if (j >= C::SB && !wait(b_sfree(sbuf), ((j / C::SB) - 1) & 1)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t a = smem_desc_sw128(sQ + (k >> 2) * (C::QB * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t bd =
              smem_desc_sw128(sK + ks * C::KV_BYTES + (k >> 2) * (P * 128) + (k & 3) * 32, 16, 1024);
          mma_bf16_ss(tmem + sbuf * P, a, bd, ID_QK, k > 0 ? 1u : 0u);
        }
        mma_commit(b_kempty(ks));
        mma_commit(b_sfull(sbuf));
      }
      // every issued MMA completes before teardown frees TMEM
      mma_commit(b_done_s);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(b_done_s, 0) && globaltimer_ns() - t0 < tmo) {}
    }
  } else if (warp == 3) {
    if (lane == 0) {
      // ================= PV issuer, kept pages in list order =================
      constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, 1);
      uint8_t* slog = prm.skip_log ? prm.skip_log + (bh * prm.num_q_blocks + qb) * prm.k_cap : nullptr;
      int cpv = 0;
      for (int i = 0; i < n_list; ++i) {
        if (!DENSE) {
          const int d = decision(i);
          if (d < 0) break;
          *pv_pos = i + 1;
          if (slog) slog[i] = d ? 0 : 1;
          if (d == 0) continue;
        }
        const int vs = cpv % C::VS, ps = cpv % C::PS;
        if (!wait(b_vfull(vs), (cpv / C::VS) & 1)) break;
        if (!wait(b_pfull(ps), (cpv / C::PS) & 1)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < P / 16; ++k) {
          const uint64_t a = smem_desc_sw128(
              sP + ps * C::P_BYTES + (k >> 2) * (C::QB * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sV + vs * C::KV_BYTES + k * 16 * 128, P * 128, 1024);
          mma_bf16_ss(tmem + C::COL_O, a, bd, ID_PV, (cpv > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(b_vempty(vs));
        mma_commit(b_pempty(ps));
        ++cpv;
      }
      mma_commit(b_done_pv);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(b_done_pv, 0) && globaltimer_ns() - t0 < tmo) {}
    }
  } else {
    // ================= softmax: two warpgroups, half a row each =================
    const int hw = (warp - 4) >> 2;      // which half of the columns
    const int q4 = warp & 3;             // TMEM lane quarter
    const int row = q4 * 32 + lane;
    const bool row_valid = row < prm.q_block;
    const int grow = row0 + row;
    const int c0 = hw * HP;              // first S column of this thread
    const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
    const bool leader = (tid == 128);
    const float sl2 = prm.scale_log2, le = prm.log2_eps;
    float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;
    int ci = 0;
    bool ok = true;     // collective: every softmax warp leaves the loop at the same page
    bool fail = false;  // this warp missed a wait after the vote; reported at the next vote
    int pid_l = 0;
    // page id of list entry j (warp-uniform); call once per j, in order
    auto page_of = [&](int j) -> int {
      if ((j & 31) == 0) pid_l = (j + lane < n_list) ? page_at(j + lane) : 0;
      return __shfl_sync(0xffffffffu, pid_l, j & 31);
    };
    // half-row max of raw logits, causal mask on the diagonal page
    auto half_max = [&](const uint32_t* src, int key0) -> float {
      float v[HP];
      if (key0 + P - 1 > row0) {  // diagonal page (warp-uniform): causal mask
#pragma unroll
        for (int e = 0; e < HP; ++e)
          v[e] = key0 + c0 + e > grow ? -INFINITY : __uint_as_float(src[e]);
      } else {
#pragma unroll
        for (int e = 0; e < HP; ++e) v[e] = __uint_as_float(src[e]);
      }
#pragma unroll
      for (int w = HP / 2; w > 0; w >>= 1)
#pragma unroll
        for (int e = 0; e < w; ++e) v[e] = fmaxf(v[e], v[e + w]);
      return v[0];
    };
    // publish the decision on page j for the V producer and the PV issuer, once
    // both are past page j - DS
    auto publish = [&](int j, bool keep) {
      if (j >= C::DS) {
        const uint64_t t0 = globaltimer_ns();
        while (min(*pv_pos, *v_pos) <= j - C::DS) {
          if (*abort_flag || globaltimer_ns() - t0 > tmo) { give_up(); break; }
          __nanosleep(32);
        }
      }
      dec_word[j % C::DS] = ((uint32_t)j << 1) | (keep ? 1u : 0u);
    };
    // kept page: online softmax with a lazily moved exponent base, then the P half
    // row (bf16) into the swizzled K-major tile of ring slot ci % PS
    auto kept_page = [&](const uint32_t* cur, float mloc, int key0) {
      const float m_new = fmaxf(m_run, mloc);
      m_run = m_new;
      const bool resc = (m_ref != -INFINITY) && (m_new > m_ref + kRescaleLog2);
      if (__any_sync(0xffffffffu, resc)) {
        // O holds earlier pages: wait for the last issued PV, rescale this half of the rows
        fail = !__all_sync(0xffffffffu,
                           wait(b_pempty((ci - 1) % C::PS), ((ci - 1) / C::PS) & 1));
        if (fail) return;
        tc_fence_after();
        const float alpha = resc ? ex2_approx(m_ref - m_new) : 1.f;
#pragma unroll 1
        for (int c = 0; c < HD / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(t_row + C::COL_O + hw * HD + c * 16, r);
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st16(t_row + C::COL_O + hw * HD + c * 16, r);
        }
        tmem_st_wait();
        l *= alpha;
      }
      if (m_new != -INFINITY && (m_ref == -INFINITY || resc)) m_ref = m_new;
      const int ps = ci % C::PS;
      if (ci >= C::PS) {
        fail = !__all_sync(0xffffffffu, wait(b_pempty(ps), ((ci / C::PS) - 1) & 1));
        if (fail) return;
      }
      const bool diag = key0 + P - 1 > row0;
      const bool rlive = row_valid && m_ref != -INFINITY;
      const float nb2 = rlive ? -m_ref : 0.f;
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t prow = sP + ps * C::P_BYTES + row * 128;
#pragma unroll
      for (int c8 = 0; c8 < HP / 8; ++c8) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i0 = c8 * 8 + 2 * e;
          float x0 = fmaf(__uint_as_float(cur[i0]), sl2, nb2);
          float x1 = fmaf(__uint_as_float(cur[i0 + 1]), sl2, nb2);
          if (!rlive || (diag && key0 + c0 + i0 > grow)) x0 = -INFINITY;
          if (!rlive || (diag && key0 + c0 + i0 + 1 > grow)) x1 = -INFINITY;
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          rs[e] += p0 + p1;
          __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
          w4[e] = *reinterpret_cast<uint32_t*>(&v2);
        }
        const int cg = (c0 >> 3) + c8;  // 16-byte chunk index within the row
        const int blk = cg >> 3, cc = cg & 7;
        st_shared_v4(prow + blk * (C::QB * 128) + ((cc ^ (row & 7)) << 4), w4[0], w4[1], w4[2],
                     w4[3]);
      }
      l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_pfull(ps));
      ++ci;
    };
    // votes of all eight softmax warps for round r of iteration it
    auto vote_round = [&](int r, int it, uint32_t bits) -> uint32_t {
      int* vt = const_cast<int*>(votes) + (r * 2 + (it & 1)) * 8;
      if (lane == 0) vt[warp - 4] = (int)bits;
      named_bar_sync(1, 256);  // orders the shared-memory exchange around it
      const int4 v0 = *reinterpret_cast<const int4*>(vt);
      const int4 v1 = *reinterpret_cast<const int4*>(vt + 4);
      return (uint32_t)(v0.x | v0.y | v0.z | v0.w | v1.x | v1.y | v1.z | v1.w);
    };
    // pages per iteration: two when a half row is 32 columns (the registers allow it)
    constexpr int BATCH = (HP == 32) ? 2 : 1;
    for (int j = 0, it = 0; j < n_list; j += BATCH, ++it) {
      const int nb = min(BATCH, n_list - j);
      int key0[BATCH];
      uint32_t sv[BATCH][HP];
      float mlh[BATCH];
      bool lv[BATCH];
#pragma unroll
      for (int t = 0; t < BATCH; ++t) key0[t] = t < nb ? page_of(j + t) * P : 0;
      // ---- S half rows of the batch: TMEM -> registers (one round trip), buffers back
      bool okw = !fail;
#pragma unroll
      for (int t = 0; t < BATCH; ++t)
        if (t < nb) okw = okw && wait(b_sfull((j + t) % C::SB), ((j + t) / C::SB) & 1);
      okw = __all_sync(0xffffffffu, okw);
      if (okw) {
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < BATCH; ++t)
          if (t < nb)
#pragma unroll
            for (int c = 0; c < HP / 32; ++c)
              tmem_ld32_async(t_row + ((j + t) % C::SB) * P + c0 + c * 32, sv[t] + c * 32);
#pragma unroll
        for (int t = 0; t < BATCH; ++t)
#pragma unroll
          for (int c = 0; c < HP / 32; ++c) {
            if (t == 0 && c == 0) tmem_ld_wait32(sv[0]);
            else reg_tie32(sv[t] + c * 32);
          }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
#pragma unroll
          for (int t = 0; t < BATCH; ++t)
            if (t < nb) mbar_arrive(b_sfree((j + t) % C::SB));
      }
      // ---- half-row maxima -> round 1 exchange
      float* hm = const_cast<float*>(hmax) + (it & 1) * 512;
#pragma unroll
      for (int t = 0; t < BATCH; ++t) {
        const float mh = (okw && t < nb) ? half_max(sv[t], key0[t]) : -INFINITY;
        lv[t] = row_valid && mh != -INFINITY;
        mlh[t] = lv[t] ? mh * sl2 : -INFINITY;
        hm[(t * 2 + hw) * 128 + row] = mlh[t];
      }
      const uint32_t all1 = vote_round(0, it, okw ? 0u : 1u);
      if (all1 & 1u) { ok = false; break; }
      float mloc[BATCH];
#pragma unroll
      for (int t = 0; t < BATCH; ++t) {
        mloc[t] = fmaxf(mlh[t], hm[(t * 2 + (hw ^ 1)) * 128 + row]);
        lv[t] = mloc[t] != -INFINITY;
      }
      // ---- round 2: votes on full row maxima.  Page j + 1 is voted for both
      // outcomes of page j, so the decisions stay exactly sequential.
      bool keep[BATCH];
      if (DENSE) {
#pragma unroll
        for (int t = 0; t < BATCH; ++t) keep[t] = true;
      } else {
        const bool n0 = lv[0] && (m_run == -INFINITY || mloc[0] - m_run >= le);
        uint32_t bits = __any_sync(0xffffffffu, n0) ? 2u : 0u;
        if (BATCH == 2 && nb == 2) {
          const float mk = fmaxf(m_run, mloc[0]);
          const bool nk = lv[BATCH - 1] && (mk == -INFINITY || mloc[BATCH - 1] - mk >= le);
          const bool ns = lv[BATCH - 1] && (m_run == -INFINITY || mloc[BATCH - 1] - m_run >= le);
          bits |= __any_sync(0xffffffffu, nk) ? 4u : 0u;
          bits |= __any_sync(0xffffffffu, ns) ? 8u : 0u;
        }
        const uint32_t all2 = vote_round(1, it, bits);
        keep[0] = (j == 0) || (all2 & 2u);
        if (BATCH == 2) keep[BATCH - 1] = keep[0] ? (all2 & 4u) != 0 : (all2 & 8u) != 0;
        if (leader)
#pragma unroll
          for (int t = 0; t < BATCH; ++t)
            if (t < nb) publish(j + t, keep[t]);
      }
#pragma unroll
      for (int t = 0; t < BATCH; ++t)
        if (t < nb && keep[t] && !fail) kept_page(sv[t], mloc[t], key0[t]);
    }
    // ---- epilogue: O / l -> bf16 (each warpgroup its half of the columns), LSE
    if (ok && !fail && ci > 0)
      fail = !__all_sync(0xffffffffu, wait(b_pempty((ci - 1) % C::PS), ((ci - 1) / C::PS) & 1));
    if (ok) {  // all softmax warps are here together: exchange the half-row sums
      hsum[hw * 128 + row] = l;
      named_bar_sync(1, 256);
      l += hsum[(hw ^ 1) * 128 + row];
    }
    tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    __nv_bfloat16* orow = prm.out + (bh * prm.seq_len + grow) * D + hw * HD;
#pragma unroll
    for (int c = 0; c < HD / 32; ++c) {
      uint32_t r[32];
      if (ok && !fail && ci > 0) {
        tmem_ld32(t_row + C::COL_O + hw * HD + c * 32, r);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = 0u;
      }
      if (row_valid) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * inv,
                                                    __uint_as_float(r[2 * e + 1]) * inv);
          w[e] = *reinterpret_cast<uint32_t*>(&v2);
        }
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
        dst[3] = make_uint4(w[12], w[13], w[14], w[15]);
      }
    }
    if (hw == 0 && row_valid && prm.lse)
      prm.lse[bh * prm.seq_len + grow] =
          l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    if (!DENSE && leader && prm.computed) prm.computed[bh * prm.num_q_blocks + qb] = ci;
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace cosa
