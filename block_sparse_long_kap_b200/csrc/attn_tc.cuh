// Ordered-Skipping Kernel (and dense causal attention) on the sm_100a tensor
// cores: TMA page loads through the page table, tcgen05.mma into TMEM, one
// softmax thread per query row.  (gist.science/pt "CoSA" technical summary,
// §2.3 "Estágio 2: OSK": mask-skipped pages are never loaded, "KV page
// remapping"; in-kernel skip from the page's local max vs the running max;
// computed pages get the full softmax + PV.)
//
// One CTA (256 threads) per (b, h_q, q-block) tile of up to 128 query rows:
//   warp 0     TMA producer: the Q tile once, then K of every listed page, in
//              list order, into a KS-stage ring (page table gives the
//              physical page; no multicast).
//   warp 1     MMA issuer (one thread): S_j = Q K_j^T into one of SB TMEM
//              buffers; once page j is decided "computed" and its P and V
//              tiles are ready, O += P_j V_j into the TMEM accumulator.  It
//              polls both streams so that a late V never stalls QK^T.
//   warp 2     TMA producer for V: loads V_j only for pages the vote keeps,
//              so a skipped page costs its K tile and one QK^T, nothing more.
//   warps 4-7  softmax, thread i <-> query row i <-> TMEM lane i: reads S_j,
//              masks the causal diagonal, takes the row max, votes on the
//              skip rule (any row with (page max - running max) >= log2 eps
//              keeps the page; the first listed page is always kept), and for
//              kept pages writes P = exp2(s - m_ref) as bf16 into a swizzled
//              shared-memory tile.  m_ref, the exponent base, moves only when
//              the running max passes it by more than 2^8 (then O and l are
//              rescaled in TMEM), which keeps the result exact.
// Every wait is bounded: on timeout the CTA records COSA_ERR_TIMEOUT in the
// status word, drains what it issued, frees TMEM and exits.
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
  static constexpr int KS = (P == 64) ? 4 : 2;    // K ring stages
  static constexpr int VS = (P == 64) ? 3 : 2;    // V ring stages
  static constexpr int PS = (P == 64) ? 3 : 2;    // P tile ring stages
  static constexpr int SB = (P == 64) ? 4 : 3;    // S buffers in TMEM
  static constexpr int DS = 16;                   // decision ring
  static constexpr uint32_t Q_BYTES = QB * D * 2;
  static constexpr uint32_t KV_BYTES = P * D * 2;
  static constexpr uint32_t P_BYTES = QB * P * 2;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KS * KV_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + VS * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_P + PS * P_BYTES;
  // q, k_full/empty, v_full/empty, s_full/free, p_full/empty, dec, vote[2], mma_done
  static constexpr int NBAR = 1 + 2 * KS + 2 * VS + 2 * SB + 2 * PS + DS + 2 + 1;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t SMEM = OFF_MISC + 128;
  static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;  // 1024-byte alignment slack
  static constexpr int COL_O = SB * P;
  static constexpr int TMEM_COLS = (SB * P + D <= 256) ? 256 : 512;
  static_assert(SB * P + D <= 512, "TMEM budget");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
};

constexpr float kRescaleLog2 = 8.0f;  // m_ref trails the running max by < 2^8

template <int D, int P, bool DENSE>
__global__ void __launch_bounds__(256, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const TcParams prm) {
  using C = TcCfg<D, P>;
  using namespace tc;
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
  auto b_dec = [&](int s) {
    return bar + 8u * (1 + 2 * C::KS + 2 * C::VS + 2 * C::SB + 2 * C::PS + s);
  };
  auto b_vote = [&](int s) { return bar + 8u * (C::NBAR - 3 + s); };
  const uint32_t b_done = bar + 8u * (C::NBAR - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sg + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + C::OFF_MISC + 4);
  volatile int* votes = reinterpret_cast<volatile int*>(sg + C::OFF_MISC + 16);     // [2][4]
  volatile int* dec_flag = reinterpret_cast<volatile int*>(sg + C::OFF_MISC + 48);  // [DS]

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
    for (int s = 0; s < C::SB; ++s) { mbar_init(b_sfull(s), 1); mbar_init(b_sfree(s), 128); }
    for (int s = 0; s < C::PS; ++s) { mbar_init(b_pfull(s), 128); mbar_init(b_pempty(s), 1); }
    for (int s = 0; s < C::DS; ++s) mbar_init(b_dec(s), 1);
    mbar_init(b_vote(0), 4);
    mbar_init(b_vote(1), 4);
    mbar_init(b_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(sb0 + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (prm.q_block < C::QB && warp >= 4) {
    // rows past the q-block are padding: zero them once (the TMA box fills the rest)
    for (int i = tid - 128; i < (C::QB - prm.q_block) * (D / 64) * 8; i += 128) {
      const int chunk = i & 7, r = prm.q_block + (i >> 3) % (C::QB - prm.q_block);
      const int kb = (i >> 3) / (C::QB - prm.q_block);
      st_shared_v4(sQ + kb * (C::QB * 128) + r * 128 + chunk * 16, 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const unsigned long long tmo = prm.timeout_ns;
  // bounded blocking wait; false on timeout or abort
  auto wait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    if (mbar_try_wait(bar_addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t spins = 0;
    while (!mbar_try_wait(bar_addr, parity)) {
      if (*abort_flag) return false;
      if ((++spins & 63u) == 0) {
        if (*(volatile int*)&g_status == COSA_ERR_TIMEOUT || globaltimer_ns() - t0 > tmo) {
          *abort_flag = 1;
          set_status(COSA_ERR_TIMEOUT);
          return false;
        }
      }
    }
    return true;
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
        if (!DENSE && i > 0) {
          ok = __all_sync(0xffffffffu, wait(b_dec(i % C::DS), (i / C::DS) & 1));
          if (!ok) break;
          if (dec_flag[i % C::DS] == 0) continue;
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
      // ================= MMA issuer =================
      constexpr uint32_t ID_QK = idesc_bf16_f32(128, P, 0);
      constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, 1);
      bool ok = wait(b_q, 0);
      tc_fence_after();
      int js = 0, ipv = 0, cpv = 0;
      uint64_t last = globaltimer_ns();
      while (ok && ipv < n_list) {
        bool prog = false;
        // ---- PV for page ipv once it is decided (and, if kept, P and V are ready)
        bool known = true, keep = true;
        if (!DENSE) {
          known = mbar_test_wait(b_dec(ipv % C::DS), (ipv / C::DS) & 1);
          keep = known && dec_flag[ipv % C::DS] != 0;
        }
        if (known) {
          if (!keep) {
            ++ipv;
            prog = true;
          } else {
            const int vs = cpv % C::VS, ps = cpv % C::PS;
            if (mbar_test_wait(b_vfull(vs), (cpv / C::VS) & 1) &&
                mbar_test_wait(b_pfull(ps), (cpv / C::PS) & 1)) {
              tc_fence_after();
#pragma unroll
              for (int k = 0; k < P / 16; ++k) {
                const uint64_t a = smem_desc_sw128(
                    sP + ps * C::P_BYTES + (k >> 2) * (C::QB * 128) + (k & 3) * 32, 16, 1024);
                const uint64_t bd =
                    smem_desc_sw128(sV + vs * C::KV_BYTES + k * 16 * 128, P * 128, 1024);
                mma_bf16_ss(tmem + C::COL_O, a, bd, ID_PV, (cpv > 0 || k > 0) ? 1u : 0u);
              }
              mma_commit(b_vempty(vs));
              mma_commit(b_pempty(ps));
              ++cpv;
              ++ipv;
              prog = true;
            }
          }
        }
        // ---- S for page js (bounded lead over the PV pointer: decision ring)
        if (js < n_list && js < ipv + C::DS - 2) {
          const int ks = js % C::KS, sbuf = js % C::SB;
          if (mbar_test_wait(b_kfull(ks), (js / C::KS) & 1) &&
              (js < C::SB || mbar_test_wait(b_sfree(sbuf), ((js / C::SB) - 1) & 1))) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint64_t a =
                  smem_desc_sw128(sQ + (k >> 2) * (C::QB * 128) + (k & 3) * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(
                  sK + ks * C::KV_BYTES + (k >> 2) * (P * 128) + (k & 3) * 32, 16, 1024);
              mma_bf16_ss(tmem + sbuf * P, a, bd, ID_QK, k > 0 ? 1u : 0u);
            }
            mma_commit(b_kempty(ks));
            mma_commit(b_sfull(sbuf));
            ++js;
            prog = true;
          }
        }
        const uint64_t now = globaltimer_ns();
        if (prog) {
          last = now;
        } else {
          if (*abort_flag) break;
          if (now - last > tmo || *(volatile int*)&g_status == COSA_ERR_TIMEOUT) {
            *abort_flag = 1;
            set_status(COSA_ERR_TIMEOUT);
            break;
          }
          __nanosleep(20);
        }
      }
      // all issued MMAs complete before teardown frees TMEM
      mma_commit(b_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(b_done, 0) && globaltimer_ns() - t0 < tmo) {}
    }
  } else if (warp >= 4) {
    // ================= softmax: thread <-> row <-> TMEM lane =================
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const bool row_valid = row < prm.q_block;
    const int grow = row0 + row;
    const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
    const bool leader = (tid == 128);
    float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;
    int ci = 0;
    bool ok = true;
    int pid_l = 0;
    for (int j = 0; j < n_list; ++j) {
      if ((j & 31) == 0) pid_l = (j + lane < n_list) ? page_at(j + lane) : 0;
      const int page = __shfl_sync(0xffffffffu, pid_l, j & 31);
      const int sbuf = j % C::SB;
      ok = __all_sync(0xffffffffu, wait(b_sfull(sbuf), (j / C::SB) & 1));
      if (!ok) break;
      tc_fence_after();
      float s[P];
#pragma unroll
      for (int c = 0; c < P / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(t_row + sbuf * P + c * 32, raw);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(raw[e]);
      }
      tc_fence_before();
      mbar_arrive(b_sfree(sbuf));
      const int key0 = page * P;
      const bool diag = key0 + P - 1 > row0;
      float mloc = -INFINITY;
#pragma unroll
      for (int c = 0; c < P; ++c) {
        float v = s[c] * prm.scale_log2;
        if (!row_valid || (diag && key0 + c > grow)) v = -INFINITY;
        s[c] = v;
        mloc = fmaxf(mloc, v);
      }
      bool skip = false;
      if (!DENSE) {
        if (j > 0) {
          const bool need =
              mloc != -INFINITY && (m_run == -INFINITY || mloc - m_run >= prm.log2_eps);
          const int any = __any_sync(0xffffffffu, need) ? 1 : 0;
          if (lane == 0) {
            votes[(j & 1) * 4 + q4] = any;
            mbar_arrive(b_vote(j & 1));
          }
          ok = __all_sync(0xffffffffu, wait(b_vote(j & 1), ((j - 1) >> 1) & 1));
          if (!ok) break;
          skip = (votes[(j & 1) * 4 + 0] | votes[(j & 1) * 4 + 1] | votes[(j & 1) * 4 + 2] |
                  votes[(j & 1) * 4 + 3]) == 0;
        }
        if (leader) {
          dec_flag[j % C::DS] = skip ? 0 : 1;
          mbar_arrive(b_dec(j % C::DS));
          if (prm.skip_log)
            prm.skip_log[(bh * prm.num_q_blocks + qb) * prm.k_cap + j] = skip ? 1 : 0;
        }
      }
      if (skip) continue;
      // ---- kept page: online softmax with a lazily moved exponent base
      const float m_new = fmaxf(m_run, mloc);
      m_run = m_new;
      const bool resc = (m_ref != -INFINITY) && (m_new > m_ref + kRescaleLog2);
      if (__any_sync(0xffffffffu, resc)) {
        // O holds earlier pages: wait for the last issued PV, rescale rows in TMEM
        ok = __all_sync(0xffffffffu, wait(b_pempty((ci - 1) % C::PS), ((ci - 1) / C::PS) & 1));
        if (!ok) break;
        tc_fence_after();
        const float alpha = resc ? exp2f(m_ref - m_new) : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_row + C::COL_O + c * 32, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(t_row + C::COL_O + c * 32, r);
        }
        tmem_st_wait();
        l *= alpha;
      }
      if (m_new != -INFINITY && (m_ref == -INFINITY || resc)) m_ref = m_new;
      // P row (bf16) into the swizzled K-major tile of ring slot ci % PS
      const int ps = ci % C::PS;
      if (ci >= C::PS) {
        ok = __all_sync(0xffffffffu, wait(b_pempty(ps), ((ci / C::PS) - 1) & 1));
        if (!ok) break;
      }
      const bool live = m_ref != -INFINITY;
      float rs = 0.f;
      const uint32_t prow = sP + ps * C::P_BYTES + row * 128;
#pragma unroll
      for (int c8 = 0; c8 < P / 8; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = live ? exp2f(s[c8 * 8 + 2 * e] - m_ref) : 0.f;
          const float p1 = live ? exp2f(s[c8 * 8 + 2 * e + 1] - m_ref) : 0.f;
          rs += p0 + p1;
          __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
          w[e] = *reinterpret_cast<uint32_t*>(&v2);
        }
        const int blk = c8 >> 3, cc = c8 & 7;
        st_shared_v4(prow + blk * (C::QB * 128) + ((cc ^ (row & 7)) << 4), w[0], w[1], w[2], w[3]);
      }
      l += rs;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(b_pfull(ps));
      ++ci;
    }
    // ---- epilogue: O / l -> bf16, LSE (natural log), computed count
    if (ok && ci > 0)
      ok = __all_sync(0xffffffffu, wait(b_pempty((ci - 1) % C::PS), ((ci - 1) / C::PS) & 1));
    tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    __nv_bfloat16* orow = prm.out + (bh * prm.seq_len + grow) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      if (ok && ci > 0) {
        tmem_ld32(t_row + C::COL_O + c * 32, r);
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
    if (row_valid && prm.lse)
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
