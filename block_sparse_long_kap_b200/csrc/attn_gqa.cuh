// Ordered-Skipping Kernel over a group-shared page list: two query heads of one
// KV head share the q-block's ordered list (cosa_kap_select_group), so each
// group of listed K pages is loaded once for both heads.  Each head keeps the
// per-head skip rule of gist.science/pt "CoSA" technical summary §2.3 ("Saltado
// no Kernel": a page is skipped when no row of the head's q-block gains from it,
// (page max - running max) < log2 eps in the log2 domain) and its own online
// softmax; the pages a head skips cost it its share of the QK^T only.
//
// One CTA (384 threads) per (b, h_kv, q-block, pair of query heads); listed
// pages go in groups of 128 keys (two pages of 64 or one of 128).
//   warp 0   Q (both heads) and K loads, TMA through the page table, no multicast
//   warp 1   MMA issue: QK0(g) QK1(g), then per head PV(g) when the head keeps a
//            page of group g, then its QK(g+1); tcgen05.mma runs in issue order,
//            so QKi(g+1) overwrites Si only after PVi(g) has read Pi(g)
//   warp 2   V loads: group g's V when either head keeps one of its pages
//   warp 3   TMEM allocation
//   warps 4-7 / 8-11  head 0 / head 1: thread = query row = TMEM lane.  Per group:
//            row max of each page, one vote round among the 128 threads for both
//            pages (the second under both outcomes of the first), then for a kept
//            group P = exp2(s * scale - m_ref) (zero on a skipped page's keys) over
//            the first 64 S columns.  The exponent base m_ref moves only when the
//            running max passes it by more than 2^32 (O and l are then rescaled in
//            TMEM; the commit that reports Si full also covers PVi(g-1)).
// The softmax of head i reports each group on an mbarrier (the MMA thread waits
// on it before touching Si again) and in a decision word (keep bits) that the
// MMA and V threads read.  Every wait is bounded: on timeout the CTA records
// COSA_ERR_TIMEOUT, drains what it issued, frees TMEM and exits.
#pragma once

#include "attn_tc.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace cosa {

template <int D, int P>
struct PairCfg {
  static constexpr int QB = 128;                   // rows per head tile (q-block padded)
  static constexpr int GP = 128 / P;               // pages per group
  static constexpr int NT = 384;
  static constexpr uint32_t Q_BYTES = QB * D * 2;
  static constexpr uint32_t PAGE_BYTES = P * D * 2;
  static constexpr uint32_t GRP_BYTES = GP * PAGE_BYTES;  // one group of K or V
  static constexpr int KS = (D == 128) ? 3 : 4;    // K ring slots (groups)
  static constexpr int VS = (D == 128) ? 2 : 4;    // V ring slots (groups)
  static constexpr int DR = 16;                    // decision ring (groups) per head
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KS * GRP_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + VS * GRP_BYTES;
  // q, k_full/empty, v_full/empty, s_full[2], g_done[2], o_full[2], done
  static constexpr int NBAR = 1 + 2 * KS + 2 * VS + 6 + 1;
  static constexpr uint32_t OFF_MISC = (OFF_BAR + NBAR * 8 + 15) & ~15u;
  // misc: +0 TMEM address, +4 abort flag, +8 decisions published [2], +16 decisions
  //       read by the V thread, +32 votes [2 heads][2 rounds][4 warps], +96 decision
  //       ring [2][DR]
  static constexpr uint32_t MISC_BYTES = 96 + 2 * DR * 4;
  static constexpr uint32_t SMEM = OFF_MISC + MISC_BYTES;
  static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int COL_O = 256;                // O of head i at COL_O + i * D
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(COL_O + 2 * D <= TMEM_COLS, "TMEM budget");
  static_assert(GRP_BYTES % 1024 == 0 && PAGE_BYTES % 1024 == 0, "1024-byte aligned tiles");
};

template <int D, int P>
__global__ void __launch_bounds__(384, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const TcParams prm) {
  using C = PairCfg<D, P>;
  using namespace tc;
  constexpr int GP = C::GP;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const uint32_t sb0 = (sraw + 1023u) & ~1023u;
  uint8_t* sg = smem_raw + (sb0 - sraw);
  const uint32_t sQ = sb0 + C::OFF_Q, sK = sb0 + C::OFF_K, sV = sb0 + C::OFF_V;
  const uint32_t bar = sb0 + C::OFF_BAR;
  const uint32_t b_q = bar;
  auto b_kfull = [&](int s) { return bar + 8u * (1 + s); };
  auto b_kempty = [&](int s) { return bar + 8u * (1 + C::KS + s); };
  auto b_vfull = [&](int s) { return bar + 8u * (1 + 2 * C::KS + s); };
  auto b_vempty = [&](int s) { return bar + 8u * (1 + 2 * C::KS + C::VS + s); };
  auto b_sfull = [&](int i) { return bar + 8u * (1 + 2 * C::KS + 2 * C::VS + i); };
  auto b_gdone = [&](int i) { return bar + 8u * (3 + 2 * C::KS + 2 * C::VS + i); };
  auto b_ofull = [&](int i) { return bar + 8u * (5 + 2 * C::KS + 2 * C::VS + i); };
  const uint32_t b_done = bar + 8u * (C::NBAR - 1);
  uint8_t* misc = sg + C::OFF_MISC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* dpub = reinterpret_cast<volatile int*>(misc + 8);    // [2]
  volatile int* vread = reinterpret_cast<volatile int*>(misc + 16);
  volatile int* votes = reinterpret_cast<volatile int*>(misc + 32);  // [2][2][4]
  volatile int* dec = reinterpret_cast<volatile int*>(misc + 96);    // [2][DR]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (__syncthreads_or(*(volatile int*)&g_status == COSA_ERR_TIMEOUT)) return;

  // ---- work decode: KV-head major, heaviest q-blocks first, head pairs fastest
  const int G = prm.group, npairs = (G + 1) / 2;
  const int per_kv = npairs * prm.num_q_blocks;
  const int z = blockIdx.x / per_kv;
  const int rem = blockIdx.x % per_kv;
  const int qb = prm.num_q_blocks - 1 - rem / npairs;
  const int pr = rem % npairs;
  const int hk = z % prm.num_kv_heads;
  const int b = z / prm.num_kv_heads;
  const int h0 = hk * G + 2 * pr;
  const bool two = 2 * pr + 1 < G;  // the pair's second head exists
  auto head = [&](int i) { return h0 + i; };
  auto active = [&](int i) { return i == 0 || two; };
  const int row0 = qb * prm.q_block;
  const int n_causal = causal_pages(qb, prm.q_block, P);
  const long long lrow = ((long long)b * prm.num_kv_heads + hk) * prm.num_q_blocks + qb;
  const int32_t* olist = prm.order + lrow * prm.k_cap;
  int n_list = min(max(prm.count[lrow], 0), prm.k_cap);
  {
    int bad = 0;
    for (int j = tid; j < n_list; j += blockDim.x) bad |= (olist[j] < 0) | (olist[j] >= n_causal);
    if (__syncthreads_or(bad)) {
      if (tid == 0) set_status(COSA_ERR_INVALID_ARG);
      n_list = 0;
    }
  }
  const int n_groups = (n_list + GP - 1) / GP;
  const int32_t* ptab = prm.page_table + (long long)b * prm.pages_per_seq;
  auto page_at = [&](int j) { return __ldg(olist + j); };
  auto coord_of = [&](int page) { return __ldg(ptab + page) * prm.num_kv_heads + hk; };
  auto pages_in = [&](int g) { return min(GP, n_list - g * GP); };

  // ---- setup
  if (tid == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < C::KS; ++s) { mbar_init(b_kfull(s), 1); mbar_init(b_kempty(s), 1); }
    for (int s = 0; s < C::VS; ++s) { mbar_init(b_vfull(s), 1); mbar_init(b_vempty(s), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_sfull(i), 1);
      mbar_init(b_gdone(i), 4);
      mbar_init(b_ofull(i), 1);
    }
    mbar_init(b_done, 1);
    *abort_flag = 0;
    dpub[0] = dpub[1] = 0;
    *vread = 0;
    fence_barrier_init();
  }
  if (warp == 3) {
    tmem_alloc(sb0 + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (prm.q_block < C::QB && warp >= 4) {
    // rows past the q-block are padding: zeros (the TMA box fills the rest)
    const int i = (warp - 4) >> 2, pad = C::QB - prm.q_block;
    for (int x = tid & 127; x < pad * (D / 64) * 8; x += 128) {
      const int chunk = x & 7, r = prm.q_block + (x >> 3) % pad, kb = (x >> 3) / pad;
      st_shared_v4(sQ + i * C::Q_BYTES + kb * (C::QB * 128) + r * 128 + chunk * 16, 0u, 0u, 0u,
                   0u);
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
  auto timed_out = [&](uint64_t t0) {
    return *(volatile int*)&g_status == COSA_ERR_TIMEOUT || globaltimer_ns() - t0 > tmo;
  };
  // bounded waits on an mbarrier phase (suspending / polling); false on timeout or abort
  auto wait = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    if (mbar_try_wait(bar_addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar_addr, parity)) {
      if (*abort_flag) return false;
      if (timed_out(t0)) {
        give_up();
        return false;
      }
    }
    return true;
  };
  auto wait_hot = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    if (mbar_test_wait(bar_addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t n = 0;
    while (!mbar_test_wait(bar_addr, parity)) {
      if ((++n & 255u) == 0) {
        if (*abort_flag) return false;
        if (timed_out(t0)) {
          give_up();
          return false;
        }
      }
    }
    return true;
  };
  auto wait_warp_hot = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    int okl = 1;
    if (lane == 0) okl = wait_hot(bar_addr, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, okl, 0) != 0;
  };
  // bounded wait (one thread) until *cnt > v; false on timeout or abort
  auto wait_count = [&](volatile int* cnt, int v) -> bool {
    if (*cnt > v) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t n = 0;
    while (*cnt <= v) {
      if ((++n & 63u) == 0) {
        if (*abort_flag) return false;
        if (timed_out(t0)) {
          give_up();
          return false;
        }
      }
    }
    return true;
  };
  // TMA loads of list group g (1 or 2 pages) into a ring slot
  auto load_group = [&](const CUtensorMap* tm, uint32_t dst, uint32_t full_bar, int g) {
    const int np = pages_in(g);
    mbar_arrive_expect_tx(full_bar, (uint32_t)np * C::PAGE_BYTES);
    for (int t = 0; t < np; ++t) {
      const int cz = coord_of(page_at(g * GP + t));
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_3d(dst + kb * (GP * P * 128) + t * (P * 128), tm, full_bar, kb * 64, 0, cz);
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      // ================= Q of both heads, then K groups in list order ============
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      const uint32_t qbytes = (uint32_t)(two ? 2 : 1) * (D / 64) * prm.q_block * 128;
      mbar_arrive_expect_tx(b_q, qbytes);
      for (int i = 0; i < 2; ++i)
        if (active(i)) {
          const int bh = b * prm.num_q_heads + head(i);
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_3d(sQ + i * C::Q_BYTES + kb * (C::QB * 128), &tm_q, b_q, kb * 64, row0, bh);
        }
      int g = 0;
      for (; g < n_groups; ++g) {
        const int s = g % C::KS;
        if (g >= C::KS && !wait(b_kempty(s), ((g / C::KS) - 1) & 1)) break;
        load_group(&tm_k, sK + s * C::GRP_BYTES, b_kfull(s), g);
      }
      // loads never consumed (abort only) land before the CTA leaves
      const uint64_t t0 = globaltimer_ns();
      drain_wait(b_q, 0, t0, tmo);
      for (int x = max(0, g - C::KS); x < g; ++x)
        drain_wait(b_kfull(x % C::KS), (x / C::KS) & 1, t0, tmo);
    }
  } else if (warp == 2) {
    if (lane == 0) {
      // ================= V of the groups some head keeps ==========================
      prefetch_tmap(&tm_v);
      int vc = 0;  // groups loaded
      bool ok = true;
      for (int g = 0; ok && g < n_groups; ++g) {
        if (!wait_count(dpub + 0, g)) break;
        int keep = dec[0 * C::DR + g % C::DR];
        if (keep == 0 && two) {
          if (!wait_count(dpub + 1, g)) break;
          keep = dec[1 * C::DR + g % C::DR];
        }
        __threadfence_block();
        *vread = g + 1;  // both decision slots of group g are read (or not needed)
        if (keep == 0) continue;
        const int s = vc % C::VS;
        if (vc >= C::VS && !wait(b_vempty(s), ((vc / C::VS) - 1) & 1)) break;
        load_group(&tm_v, sV + s * C::GRP_BYTES, b_vfull(s), g);
        ++vc;
      }
      const uint64_t t0 = globaltimer_ns();
      for (int x = max(0, vc - C::VS); x < vc; ++x)
        drain_wait(b_vfull(x % C::VS), (x / C::VS) & 1, t0, tmo);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================= MMA issue ================================================
      constexpr uint32_t ID_QK = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t ID_QK64 = idesc_bf16_f32(128, 64, 0);  // a lone last 64-key page
      constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, 1);
      // tile bases; a 16-byte aligned offset below 256 KB adds to the start-address field
      const uint64_t dq = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dk = smem_desc_sw128(sK, 16, 1024);
      const uint64_t dv = smem_desc_sw128(sV, GP * P * 128, 1024);
      // S_i = Q_i K_g^T
      auto qk = [&](int i, int g) {
        const uint32_t id = pages_in(g) * P == 128 ? ID_QK : ID_QK64;
        const uint64_t dqi = dq + ((uint32_t)i * C::Q_BYTES >> 4);
        const uint64_t dks = dk + ((uint32_t)(g % C::KS) * C::GRP_BYTES >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_ss(tmem + i * 128, dqi + (((k >> 2) * (C::QB * 128) + (k & 3) * 32) >> 4),
                      dks + (((k >> 2) * (GP * P * 128) + (k & 3) * 32) >> 4), id, k > 0 ? 1u : 0u);
        mma_commit(b_sfull(i));
      };
      // O_i += P_i V_g, P_i from TMEM (16 keys per step = 8 columns)
      auto pv = [&](int i, int g, int vs, bool first) {
        const uint64_t dvs = dv + ((uint32_t)vs * C::GRP_BYTES >> 4);
        const int nk = pages_in(g) * P / 16;
        for (int k = 0; k < nk; ++k)
          mma_bf16_ts(tmem + C::COL_O + i * D, tmem + i * 128 + k * 8, dvs + ((k * 16 * 128) >> 4),
                      ID_PV, (!first || k > 0) ? 1u : 0u);
      };
      bool ok = n_groups > 0 && wait(b_q, 0) && wait(b_kfull(0), 0);
      if (ok) {
        tc_fence_after();
        for (int i = 0; i < 2; ++i)
          if (active(i)) qk(i, 0);
        mma_commit(b_kempty(0));
      }
      bool first[2] = {true, true};
      int vc = 0;  // V groups consumed
      for (int g = 0; ok && g < n_groups; ++g) {
        const int vs = vc % C::VS;
        bool needed = false, k_next = false;
        for (int i = 0; i < 2 && ok; ++i) {
          if (!active(i)) continue;
          // head i is done with S_i for group g (read, and P written when kept)
          if (!wait_hot(b_gdone(i), g & 1)) { ok = false; break; }
          tc_fence_after();
          const int keep = dec[i * C::DR + g % C::DR];
          if (keep != 0) {
            if (!needed && !wait(b_vfull(vs), (vc / C::VS) & 1)) { ok = false; break; }
            needed = true;
            tc_fence_after();
            pv(i, g, vs, first[i]);
            first[i] = false;
          }
          if (g + 1 < n_groups) {
            if (!k_next) {
              if (!wait(b_kfull((g + 1) % C::KS), ((g + 1) / C::KS) & 1)) { ok = false; break; }
              tc_fence_after();
              k_next = true;
            }
            qk(i, g + 1);
            if (i == 1 || !two) mma_commit(b_kempty((g + 1) % C::KS));  // last reader of K(g+1)
          } else {
            mma_commit(b_ofull(i));
          }
        }
        if (!ok) break;
        if (needed) {
          mma_commit(b_vempty(vs));
          ++vc;
        }
      }
      // every issued MMA completes before teardown frees TMEM
      mma_commit(b_done);
      const uint64_t t0 = globaltimer_ns();
      drain_wait(b_done, 0, t0, tmo);
    }
  } else if (warp >= 4 && active((warp - 4) >> 2)) {
    // ================= softmax of head i, one query row per thread ==================
    const int i = (warp - 4) >> 2, q4 = warp & 3, row = q4 * 32 + lane;
    const bool row_valid = row < prm.q_block;
    const int grow = row0 + row;
    const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t t_s = t_row + i * 128, t_o = t_row + C::COL_O + i * D;
    const bool leader = q4 == 0 && lane == 0;
    const float sl2 = prm.scale_log2, le = prm.log2_eps;
    const long long bh = (long long)b * prm.num_q_heads + head(i);
    uint8_t* slog = prm.skip_log ? prm.skip_log + (bh * prm.num_q_blocks + qb) * prm.k_cap : nullptr;
    float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;  // log2 domain, base m_ref
    int n_kept = 0;
    bool ok = true;
    for (int g = 0; g < n_groups; ++g) {
      const int j0 = g * GP, nb = pages_in(g);
      int key0[GP];
#pragma unroll
      for (int t = 0; t < GP; ++t) key0[t] = t < nb ? page_at(j0 + t) * P : 0;
      const bool okw = wait_warp_hot(b_sfull(i), g & 1);
      if (okw) tc_fence_after();
      // ---- row maxima of the group's pages (raw logits; causal mask on diagonal pages)
      float mloc[GP];
      bool lv[GP];
#pragma unroll
      for (int t = 0; t < GP; ++t) {
        float mx = -INFINITY;
        if (okw && t < nb) {
#pragma unroll 1
          for (int c = 0; c < P / 64; ++c) {
            uint32_t v[64];
            tmem_ld64(t_s + t * P + c * 64, v);
            const int k0 = key0[t] + c * 64;
            if (k0 + 63 > row0) {  // a diagonal page (warp-uniform)
#pragma unroll
              for (int e = 0; e < 64; ++e)
                if (k0 + e > grow) v[e] = __float_as_uint(-INFINITY);
            }
            float a[8];
#pragma unroll
            for (int e = 0; e < 64; ++e)
              a[e & 7] = e < 8 ? __uint_as_float(v[e]) : fmaxf(a[e & 7], __uint_as_float(v[e]));
#pragma unroll
            for (int w = 4; w > 0; w >>= 1)
#pragma unroll
              for (int e = 0; e < w; ++e) a[e] = fmaxf(a[e], a[e + w]);
            mx = fmaxf(mx, a[0]);
          }
        }
        const float mr = row_valid ? mx : -INFINITY;
        lv[t] = mr != -INFINITY;
        mloc[t] = lv[t] ? mr * sl2 : -INFINITY;
      }
      // ---- votes of the group's pages against the running max: page 1 (2), page 2
      // after page 1 kept (4), page 2 after page 1 skipped (8); 1 = a failed wait
      uint32_t bits = okw ? 0u : 1u;
      {
        const bool n0 = lv[0] && (m_run == -INFINITY || mloc[0] - m_run >= le);
        bits |= __any_sync(0xffffffffu, n0) ? 2u : 0u;
        if (GP == 2 && nb == 2) {
          const float mk = fmaxf(m_run, mloc[0]);
          const bool nk = lv[GP - 1] && (mk == -INFINITY || mloc[GP - 1] - mk >= le);
          const bool ns = lv[GP - 1] && (m_run == -INFINITY || mloc[GP - 1] - m_run >= le);
          bits |= __any_sync(0xffffffffu, nk) ? 4u : 0u;
          bits |= __any_sync(0xffffffffu, ns) ? 8u : 0u;
        }
      }
      int* vt = const_cast<int*>(votes) + (i * 2 + (g & 1)) * 4;
      if (lane == 0) vt[q4] = (int)bits;
      named_bar_sync(1 + i, 128);
      const int4 vv = *reinterpret_cast<const int4*>(vt);
      const uint32_t all = (uint32_t)(vv.x | vv.y | vv.z | vv.w);
      if (all & 1u) { ok = false; break; }
      bool keep[GP];
      keep[0] = (j0 == 0) || (all & 2u);
      if (GP == 2) keep[GP - 1] = nb == 2 && (keep[0] ? (all & 4u) != 0 : (all & 8u) != 0);
      // ---- running max, and the exponent base (one base for the whole group)
      const float m_ref_old = m_ref;
      int kbits = 0;
#pragma unroll
      for (int t = 0; t < GP; ++t)
        if (t < nb && keep[t]) {
          kbits |= 1 << t;
          const float m_new = fmaxf(m_run, mloc[t]);
          m_run = m_new;
          const bool resc = (m_ref != -INFINITY) && (m_new > m_ref + kRescaleLog2);
          if (m_new != -INFINITY && (m_ref == -INFINITY || resc)) m_ref = m_new;
        }
      if (kbits != 0) {
        // the base moved for some row of this warp: O (at rest: the commit that
        // reported S_i full covers PV_i of the group before) and l to the new base
        const bool moved = m_ref_old != -INFINITY && m_ref != m_ref_old;
        if (__any_sync(0xffffffffu, moved)) {
          const float alpha = moved ? ex2_approx(m_ref_old - m_ref) : 1.f;
#pragma unroll 1
          for (int k = 0; k < D / 16; ++k) {
            uint32_t r[16];
            tmem_ld16(t_o + k * 16, r);
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st16(t_o + k * 16, r);
          }
          tmem_st_wait();
          l *= alpha;
        }
        // ---- P = exp2(s * scale - m_ref) (bf16 pairs): S columns [64c, 64c + 64) give
        // P columns [32c, 32c + 32), already read; zero on a skipped page
        const bool rlive = row_valid && m_ref != -INFINITY;
        const float nb2 = rlive ? -m_ref : 0.f;
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int c = 0; c < nb * P / 64; ++c) {
          const int t = c * 64 / P;
          const bool kt = (kbits >> t) & 1;
          const int k0 = key0[t == 0 ? 0 : GP - 1] + (c * 64 - t * P);
          const bool diag = k0 + 63 > row0;
          uint32_t cur[64];
          tmem_ld64(t_s + c * 64, cur);
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int i0 = h2 * 32 + 2 * e, key = k0 + i0;
              float x0 = fmaf(__uint_as_float(cur[i0]), sl2, nb2);
              float x1 = fmaf(__uint_as_float(cur[i0 + 1]), sl2, nb2);
              if (!rlive || !kt || (diag && key > grow)) x0 = -INFINITY;
              if (!rlive || !kt || (diag && key + 1 > grow)) x1 = -INFINITY;
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              rs[e & 3] += p0 + p1;
              __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
              w[e] = *reinterpret_cast<uint32_t*>(&v2);
            }
            tmem_st16(t_s + c * 32 + h2 * 16, w);
          }
        }
        l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
        tmem_st_wait();
      }
      // ---- the decision, then group g is reported done
      if (leader) {
        // decision slot g % DR: the V thread has read the group DR before it
        bool fine = g < C::DR || wait_count(vread, g - C::DR);
        dec[i * C::DR + g % C::DR] = kbits;
        __threadfence_block();
        dpub[i] = g + 1;
        if (slog)
          for (int t = 0; t < nb; ++t) slog[j0 + t] = ((kbits >> t) & 1) ? 0 : 1;
        (void)fine;  // a failed wait has set the abort flag: every later wait returns
      }
      n_kept += __popc(kbits);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_gdone(i));
    }
    // ---- epilogue: O / l -> bf16, LSE, pages computed
    int hv = 0;
    if (lane == 0) hv = (ok && n_groups > 0 && *abort_flag == 0) ? 1 : 0;
    bool have = __shfl_sync(0xffffffffu, hv, 0) != 0;
    if (have) have = wait_warp_hot(b_ofull(i), 0);
    tc_fence_after();
    const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
    __nv_bfloat16* orow = prm.out + (bh * prm.seq_len + grow) * D;
#pragma unroll 1
    for (int k = 0; k < D / 32; ++k) {
      uint32_t r[32];
      if (have) {
        tmem_ld32(t_o + k * 32, r);
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
        uint4* dst = reinterpret_cast<uint4*>(orow + k * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
        dst[3] = make_uint4(w[12], w[13], w[14], w[15]);
      }
    }
    if (row_valid && prm.lse)
      prm.lse[bh * prm.seq_len + grow] =
          (have && l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    if (leader && prm.computed) prm.computed[bh * prm.num_q_blocks + qb] = n_kept;
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace cosa
