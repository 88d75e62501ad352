// Ordered-Skipping Kernel on the sm_100a tensor cores: TMA page loads through the page table, tcgen05.mma into TMEM, one
// query row per TMEM lane.  (gist.science/pt "CoSA" technical summary,
// §2.3 "Estágio 2: OSK": mask-skipped pages are never loaded, "KV page
// remapping"; in-kernel skip from the page's local max vs the running max;
// computed pages get the full softmax + PV.)
//
// One CTA (384 threads) per (b, h_q, q-block) tile of up to 128 query rows.
// Listed pages are taken in list order in groups of 128 keys (two pages of 64
// keys, or one of 128): one QK^T of N = 128 per group, into one of three S
// buffers in TMEM.
//   warp 0 (1)  Q and K loads: group g into ring slot g % KG; warp 0 loads every
//               group when there are two QK^T issuers, else warps 0 and 1 take
//               the groups in turn.  The physical page comes from the page table,
//               looked up ahead of the copies; no multicast.
//   warp 2      V loads and PV (one thread): loads V of the kept pages only,
//               once the vote has kept them (up to VS pages ahead), so a skipped
//               page costs its K tile and its share of one QK^T, nothing more;
//               then O += P_c V_c with P read from TMEM.
//   warps 3, 1  QK^T issuers (one thread each): warp 3 the even groups and warp 1
//               the odd ones (warp 3 all of them when KG is odd); warp 3 also
//               allocates TMEM.  An MMA issue blocks its thread until the tensor
//               core's short queue has room, so what a thread does between two
//               groups (barrier tests, ring positions) leaves the tensor core
//               idle unless another thread's MMAs are queued.
// Barrier phases are waited on by parity, which only tells a phase from the one
// before it: a waiter must have seen the previous phase of the same barrier
// complete.  With two issuers the groups no longer complete in order, so the S
// buffer barriers are kept per group parity: group g reports S full on
// s_full[g % 3][g % 2], and the group that reuses its buffer (g + 3, the other
// parity) waits on s_free[g % 3][(g + 1) % 2]; each barrier then serves one
// thread's groups in order, 6 groups apart.  A K slot serves groups of one
// parity when KG is even, which is why a single issuer is kept when it is odd.
//   warps 4-7,  softmax, two warpgroups taking the groups in turn (even groups
//   8-11        warpgroup 0, odd groups warpgroup 1).  Thread (warp % 4, lane)
//               owns query row 32 (warp % 4) + lane, which is its TMEM lane,
//               and reads the whole row of S.  The skip rule "page j is skipped
//               when no row has (page max - running max) >= log2 eps" is first
//               voted against the running max this warpgroup last saw: the
//               running max only grows, so a page skipped against an older
//               value is skipped against the current one, and an all-skip group
//               is settled without waiting for the other warpgroup.  A group
//               with a page that may be kept (and the first group) waits until the groups before it are
//               settled, reads the exact running max and exponent base of every
//               row from shared memory and votes again; its pages are then
//               published in list order.  One barrier round among the 128
//               threads of a warpgroup carries each vote, for the group's second
//               page under both outcomes of the first.  The first listed page is
//               always kept.  For kept pages each thread writes
//               P = exp2(s - m_ref) (bf16) for its row over the page's S
//               columns; m_ref, the exponent base, moves only when the running
//               max passes it by more than 2^32 (O and l are then rescaled),
//               which keeps the result exact: P <= 2^32 stays well inside the
//               range of bf16, and l and O inside fp32.
// Kept pages reach the V/PV thread through a shared-memory
// queue that carries each page's TMA coordinate and P location; the
// consumers' progress counters give it back-pressure.  Every wait is bounded: on
// timeout the CTA records COSA_ERR_TIMEOUT in the status word, drains what it
// issued, frees TMEM and exits; a timed-out CTA makes every later CTA of the
// launch exit at once.
// Optional early break (max_run = r > 0, not part of the pages' method): a page with
// r skipped pages right before it, and every page after it, is skipped unvisited.  The
// exact path applies this page by page from the list position of the last kept page;
// a stop group index, lowered once the break is proven from settled groups, ends the
// K loads, the QK^T issue and the softmax loop early, and every wait that could be for
// a group past it gives up.
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
  int max_run;  // OSK early break after this many consecutive skipped pages; 0: none
  unsigned long long timeout_ns;
  int fault_k_group;  // test hook: the K copies of this listed group are never issued (-1: none)
};

template <int D, int P>
struct TcCfg {
  static constexpr int QB = 128;                  // MMA M (rows per tile, padded)
  static constexpr int NT = 384;                  // 12 warps
  static constexpr int GP = 128 / P;              // pages per QK group (128 keys)
  static constexpr uint32_t Q_BYTES = QB * D * 2;
  static constexpr uint32_t KV_BYTES = P * D * 2; // one page of K or of V
  static constexpr uint32_t KG_BYTES = GP * KV_BYTES;
  // Shared memory goes to the K ring first: every group streams K, only kept pages
  // stream V.  D = 128, P = 64: Q 32 KB + K 4 x 32 KB + V 2 x 16 KB = 192 KB;
  // P = 128: Q 32 KB + K 3 x 32 KB + V 2 x 32 KB = 192 KB; D = 64: 16 + 96 + 32 KB.
  static constexpr int KG = (D == 128) ? (P == 64 ? 4 : 3) : 6;  // K ring slots (groups)
  static constexpr int VS = (P == 64 || D == 64) ? (int)(32768u / KV_BYTES) : 2;  // V slots
  static constexpr int SBG = 3;                   // S group buffers in TMEM, 128 columns each
  static constexpr bool TWO_QK = KG % 2 == 0;     // two QK^T issuers (K slots of one parity)
  static constexpr int NPROD = TWO_QK ? 1 : 2;     // K producer warps (warp 1 when free)
  static constexpr int COL_O = SBG * 128;         // O accumulator (D columns)
  static constexpr int PF = 8;                    // P-ready barrier ring (kept pages)
  static constexpr int PD = 8;                    // PV-done barrier ring (kept pages)
  static constexpr int KQ = 64;                   // kept-page queue entries
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KG * KG_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + VS * KV_BYTES;
  // q, k_full/empty, v_full/empty, s_full/free [SBG][2], p_full, pv_done, done (QK even, odd), done (PV)
  static constexpr int NBAR = 1 + 2 * KG + 2 * VS + 4 * SBG + PF + PD + 3;
  static constexpr uint32_t OFF_MISC = (OFF_BAR + NBAR * 8 + 127) & ~127u;  // vector-aligned
  // misc: +0 TMEM address, +4 abort flag, +8 kept count (P location published),
  //       +12 final kept count (-1 while the votes run), +16 V progress,
  //       +20 warpgroups finished, +24 first group past an early break, +28 list
  //       position of the last kept page, +36 PV progress, +40 kept count (TMA coordinate
  //       published), +48 votes [2 wg][2][4], +128 kept queue [KQ] {TMA coordinate,
  //       P column | last << 15}, +640 settled state rows [128] {m_run, m_ref},
  //       +1664 last settled group per softmax warp [8], +1696 S-ready flag per
  //       warpgroup [2], +1704 last group loaded per K producer warp [2],
  //       +2688 final rows [2][128] {l, m_ref}
  static constexpr uint32_t M_STATE = 640, M_SETTLED = 1664, M_FIN = 2688;
  static constexpr uint32_t MISC_BYTES = M_FIN + 2 * 128 * 8;
  static constexpr uint32_t SMEM = OFF_MISC + MISC_BYTES;
  static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;  // 1024-byte alignment slack
  static_assert(COL_O + D <= TMEM_COLS, "TMEM budget");
  static_assert(VS >= 2 && KG >= 2, "ring depths");
  static_assert(SBG % 2 == 1, "S buffer barriers per group parity: 2 * SBG groups apart");
  static_assert(PF >= 2 * SBG + 1 && PD >= 2 * SBG + 1, "barrier rings cover the kept pages in flight");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(OFF_MISC % 128 == 0, "16-byte vector access to the vote words");
  static_assert(KV_BYTES % 1024 == 0, "tiles stay 1024-byte aligned for the 128-byte swizzle");
  static_assert(48 + 64 <= 128 && 128 + 8 * KQ <= M_STATE, "vote words and kept queue fit");
  static_assert(M_STATE + 128 * 8 <= M_SETTLED && M_SETTLED + 8 * 4 + 4 * 4 <= M_FIN,
                "state rows and flags fit");
};

// m_ref trails the running max by < 2^32: a rescale waits for the PV before it,
// so it is kept rare; P = exp2(s - m_ref) <= 2^32, l <= 2^32 * keys, all in range
constexpr float kRescaleLog2 = 32.0f;

// BRK: the early break is compiled in (max_run > 0); without it the kernel carries none
// of its code, which keeps the hot loop's instruction footprint small
template <int D, int P, bool BRK>
__global__ void __launch_bounds__(TcCfg<D, P>::NT, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const TcParams prm) {
  using C = TcCfg<D, P>;
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
  auto b_kempty = [&](int s) { return bar + 8u * (1 + C::KG + s); };
  auto b_vfull = [&](int s) { return bar + 8u * (1 + 2 * C::KG + s); };
  auto b_vempty = [&](int s) { return bar + 8u * (1 + 2 * C::KG + C::VS + s); };
  // S buffer s, group parity p (see the note on barrier phases above)
  auto b_sfull = [&](int s, int p) { return bar + 8u * (1 + 2 * C::KG + 2 * C::VS + 2 * s + p); };
  auto b_sfree = [&](int s, int p) {
    return bar + 8u * (1 + 2 * C::KG + 2 * C::VS + 2 * C::SBG + 2 * s + p);
  };
  auto b_pfull = [&](int s) { return bar + 8u * (1 + 2 * C::KG + 2 * C::VS + 4 * C::SBG + s); };
  auto b_pvdone = [&](int s) {
    return bar + 8u * (1 + 2 * C::KG + 2 * C::VS + 4 * C::SBG + C::PF + s);
  };
  const uint32_t b_done = bar + 8u * (C::NBAR - 3);      // QK^T, even groups
  const uint32_t b_done_odd = bar + 8u * (C::NBAR - 2);  // QK^T, odd groups
  const uint32_t b_done_pv = bar + 8u * (C::NBAR - 1);
  uint8_t* misc = sg + C::OFF_MISC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* kq_count = reinterpret_cast<volatile int*>(misc + 8);
  volatile int* kq_final = reinterpret_cast<volatile int*>(misc + 12);
  volatile int* v_pos = reinterpret_cast<volatile int*>(misc + 16);
  int* wg_done = reinterpret_cast<int*>(misc + 20);
  // early break (max_run > 0): groups >= *stop_g lie past it; *kept_last is the list
  // position of the last kept page, written in list order by the exact path
  volatile int* stop_g = reinterpret_cast<volatile int*>(misc + 24);
  volatile int* kept_last = reinterpret_cast<volatile int*>(misc + 28);
  volatile int* pv_pos = reinterpret_cast<volatile int*>(misc + 36);
  volatile int* vq_count = reinterpret_cast<volatile int*>(misc + 40);
  volatile int* votes = reinterpret_cast<volatile int*>(misc + 48);     // [2][2][4]
  volatile int* settled = reinterpret_cast<volatile int*>(misc + C::M_SETTLED);  // [8]
  volatile int* s_ok = reinterpret_cast<volatile int*>(misc + C::M_SETTLED + 32);  // [2]
  // last group each K producer warp loaded (for the drain after an early break)
  volatile int* k_last = reinterpret_cast<volatile int*>(misc + C::M_SETTLED + 40);  // [2]
  volatile int2* kq = reinterpret_cast<volatile int2*>(misc + 128);     // [KQ]
  volatile float2* st_rows = reinterpret_cast<volatile float2*>(misc + C::M_STATE);  // [128]
  volatile float2* fin_rows = reinterpret_cast<volatile float2*>(misc + C::M_FIN);    // [2][128]

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
  {
    olist = prm.order + (bh * prm.num_q_blocks + qb) * prm.k_cap;
    n_list = min(max(prm.count[bh * prm.num_q_blocks + qb], 0), prm.k_cap);
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
  // TMA z coordinate of a logical page in the [phys page][kv head] pools
  auto coord_of = [&](int page) { return __ldg(ptab + page) * prm.num_kv_heads + hk; };

  // ---- setup
  if (tid == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < C::KG; ++s) { mbar_init(b_kfull(s), 1); mbar_init(b_kempty(s), 1); }
    for (int s = 0; s < C::VS; ++s) { mbar_init(b_vfull(s), 1); mbar_init(b_vempty(s), 1); }
    for (int s = 0; s < C::SBG; ++s)
      for (int p = 0; p < 2; ++p) { mbar_init(b_sfull(s, p), 1); mbar_init(b_sfree(s, p), 1); }
    for (int s = 0; s < C::PF; ++s) mbar_init(b_pfull(s), 4);
    for (int s = 0; s < C::PD; ++s) mbar_init(b_pvdone(s), 1);
    mbar_init(b_done, 1);
    mbar_init(b_done_odd, 1);
    mbar_init(b_done_pv, 1);
    *abort_flag = 0;
    *kq_count = 0;
    *kq_final = -1;
    *v_pos = 0;
    *pv_pos = 0;
    *vq_count = 0;
    *wg_done = 0;
    *stop_g = n_groups;
    *kept_last = -1;
    k_last[0] = -1;
    k_last[1] = -1;
    for (int w = 0; w < 8; ++w) settled[w] = -1;
    for (int r = 0; r < 128; ++r) {
      st_rows[r].x = -INFINITY;
      st_rows[r].y = -INFINITY;
    }
    fence_barrier_init();
  }
  if (warp == 3) {
    tmem_alloc(sb0 + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (prm.q_block < C::QB && warp >= 4 && warp < 8) {
    // rows past the q-block are padding: zero them once (the TMA box fills the rest)
    const int pad = C::QB - prm.q_block;
    for (int i = tid - 128; i < pad * (D / 64) * 8; i += 128) {
      const int chunk = i & 7, r = prm.q_block + (i >> 3) % pad, kb = (i >> 3) / pad;
      st_shared_v4(sQ + kb * (C::QB * 128) + r * 128 + chunk * 16, 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const unsigned long long tmo = prm.timeout_ns;
  const int R = BRK ? prm.max_run : 0;  // early break after R consecutive skipped pages (0: none)
  auto give_up = [&]() {
    *abort_flag = 1;
    set_status(COSA_ERR_TIMEOUT);
  };
  auto timed_out = [&](uint64_t t0) {
    return *(volatile int*)&g_status == COSA_ERR_TIMEOUT || globaltimer_ns() - t0 > tmo;
  };
  // bounded blocking wait on an mbarrier phase; false on timeout or abort
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
  // the same for work of group g: 1 done, 0 timeout or abort, 2 group g now lies past an
  // early break (the phase may never complete: nothing past the break is loaded or issued)
  auto wait_g = [&](uint32_t bar_addr, uint32_t parity, int g) -> int {
    if (mbar_try_wait(bar_addr, parity)) return 1;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar_addr, parity)) {
      if (g >= *stop_g) return 2;
      if (*abort_flag) return 0;
      if (timed_out(t0)) {
        give_up();
        return 0;
      }
    }
    return 1;
  };
  // the same, waited on by lane 0 for the whole warp
  auto wait_warp = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    int okl = 1;
    if (lane == 0) okl = wait(bar_addr, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, okl, 0) != 0;
  };

  // bounded wait (one thread) until counter cnt passes kept page c: 1 = it exists,
  // 0 = the list ended before it, -1 = abort
  auto kept_ready = [&](volatile int* cnt, int c) -> int {
    if (*cnt > c) return 1;
    const uint64_t t0 = globaltimer_ns();
    uint32_t spins = 0, nap = 64;
    while (true) {
      const int f = *kq_final;
      if (*cnt > c) return 1;
      if (f >= 0) return 0;
      if (*abort_flag) return -1;
      if ((++spins & 15u) == 0 && timed_out(t0)) {
        give_up();
        return -1;
      }
      __nanosleep(nap);
      nap = min(nap * 2, 512u);
    }
  };

  if (warp < C::NPROD) {
    // ================= Q (warp 0), then K: groups g = warp, warp + NPROD, ... ========
    const int kp = warp;
    if (kp == 0 && lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      mbar_arrive_expect_tx(b_q, (uint32_t)((D / 64) * prm.q_block * 128));
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_3d(sQ + kb * (C::QB * 128), &tm_q, b_q, kb * 64, row0, (int)bh);
    }
    int last = -1;  // last group this warp issued
    bool ok = true;
    constexpr int GB = 32 / GP;  // this warp's groups per block of page-table lookups
    // lane l: the logical page of page l % GP of this warp's group i0 + l / GP (-1 past
    // the list).  Page ids are read two blocks ahead and TMA coordinates one block
    // ahead, so the copies never wait on those global loads.
    auto page_of_lane = [&](int i0) -> int {
      const int jl = (kp + C::NPROD * (i0 + lane / GP)) * GP + lane % GP;
      return jl < n_list ? page_at(jl) : -1;
    };
    const int n_mine = (n_groups - kp + C::NPROD - 1) / C::NPROD;  // this warp's groups
    int cz_next;
    {
      const int pg0 = page_of_lane(0);
      cz_next = pg0 >= 0 ? coord_of(pg0) : 0;
    }
    int pg_next = GB < n_mine ? page_of_lane(GB) : -1;
    for (int i0 = 0; ok && i0 < n_mine; i0 += GB) {
      const int cz_l = cz_next;
      cz_next = pg_next >= 0 ? coord_of(pg_next) : 0;
      pg_next = i0 + 2 * GB < n_mine ? page_of_lane(i0 + 2 * GB) : -1;
      for (int mm = 0; mm < GB; ++mm) {
        const int g = kp + C::NPROD * (i0 + mm);
        if (g >= n_groups) break;
        // nothing past an early break is loaded (one read for the warp; none without a
        // break, where the stop never moves)
        if (R > 0 && __shfl_sync(0xffffffffu, lane == 0 ? *stop_g : 0, 0) <= g) {
          ok = false;
          break;
        }
        const int s = g % C::KG;
        if (g >= C::KG) {
          int r = 1;
          if (lane == 0) r = wait_g(b_kempty(s), ((g / C::KG) - 1) & 1, g);
          if (__shfl_sync(0xffffffffu, r, 0) != 1) {
            ok = false;
            break;
          }
        }
        const int nb = min(GP, n_list - g * GP);
        int cz[GP];
#pragma unroll
        for (int t = 0; t < GP; ++t) cz[t] = __shfl_sync(0xffffffffu, cz_l, mm * GP + t);
        // test hook: a withheld group's copies never arrive, so its waits run out
        const bool withhold = g == prm.fault_k_group;
        // lane 0 posts the group's bytes, then lane t copies page t: copies issued from
        // separate threads stream side by side
        if (lane == 0 && !withhold) mbar_arrive_expect_tx(b_kfull(s), (uint32_t)nb * C::KV_BYTES);
        __syncwarp();
        if (lane < nb && !withhold) {
          const int czt = (GP == 2 && lane == 1) ? cz[GP - 1] : cz[0];
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_3d(sK + s * C::KG_BYTES + kb * (GP * P * 128) + lane * (P * 128), &tm_k,
                        b_kfull(s), kb * 64, 0, czt);
        }
        last = g;
        __syncwarp();
      }
    }
    if (lane == 0) k_last[kp] = last;
    if (lane == 0 && *abort_flag) {  // drain what was issued and never consumed
      const uint64_t t0 = globaltimer_ns();
      if (kp == 0)
        drain_wait(b_q, 0, t0, tmo);
      for (int g = last; g >= 0 && g > last - C::NPROD * C::KG; g -= C::NPROD)
        if (g != prm.fault_k_group) drain_wait(b_kfull(g % C::KG), (g / C::KG) & 1, t0, tmo);
    }
  } else if (warp == 2) {
    if (lane == 0) {
      // ================= V loads and PV, kept pages in list order =================
      // V tiles are loaded ahead (up to VS pages) as the kept pages become known;
      // PV of page c follows once its P and V are in place.
      prefetch_tmap(&tm_v);
      constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, 1);
      const uint64_t dv = smem_desc_sw128(sV, P * 128, 1024);
      int nv = 0;                          // V loads issued
      int c = 0;                           // PV issued
      int pv_end = -1;                     // kept pages in all (once known)
      bool ok = true;
      // issue the V load of kept page nv (its slot is free)
      auto load_v = [&]() {
        __threadfence_block();
        const int cz = kq[nv % C::KQ].x;
        *v_pos = nv + 1;  // queue entry nv has been read
        const int s = nv % C::VS;
        mbar_arrive_expect_tx(b_vfull(s), C::KV_BYTES);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_3d(sV + s * C::KV_BYTES + kb * (P * 128), &tm_v, b_vfull(s), kb * 64, 0, cz);
        ++nv;
      };
      auto v_known = [&](int x) { return *vq_count > x; };
      while (ok) {
        // ---- kept page c known (or the list ended)?
        if (pv_end < 0) {
          const int r = kept_ready(kq_count, c);
          if (r < 0) break;
          if (r == 0) pv_end = *kq_final;
        }
        if (pv_end >= 0 && c >= pv_end) break;
        // ---- its V, and the following ones while slots are free (no waiting)
        if (nv == c) {
          if (c >= C::VS && !wait(b_vempty(c % C::VS), ((c / C::VS) - 1) & 1)) break;
          load_v();
        }
        while (nv < c + C::VS && v_known(nv) &&
               (nv < C::VS || mbar_test_wait(b_vempty(nv % C::VS), ((nv / C::VS) - 1) & 1)))
          load_v();
        // ---- PV of page c
        __threadfence_block();
        const int info = kq[c % C::KQ].y;
        const int col = info & 0x7fff, lastg = (info >> 15) & 1, gpar = (info >> 16) & 1;
        const int vs = c % C::VS;
        if (!wait(b_vfull(vs), (c / C::VS) & 1)) break;
        if (!wait(b_pfull(c % C::PF), (c / C::PF) & 1)) break;
        tc_fence_after();
        const uint64_t dvs = dv + ((uint32_t)vs * C::KV_BYTES >> 4);
#pragma unroll
        for (int k = 0; k < P / 16; ++k)
          mma_bf16_ts(tmem + C::COL_O, tmem + col + k * 8, dvs + ((k * 16 * 128) >> 4), ID_PV,
                      (c > 0 || k > 0) ? 1u : 0u);
        mma_commit(b_vempty(vs));
        mma_commit(b_pvdone(c % C::PD));
        // the group's S buffer goes back, to the issuer of the group that reuses it
        if (lastg) mma_commit(b_sfree(col >> 7, gpar ^ 1));
        ++c;
        *pv_pos = c;  // queue entry c - 1 has been read
      }
      // every issued PV completes before teardown frees TMEM; V loads never consumed
      // (abort only) land before the CTA leaves
      mma_commit(b_done_pv);
      const uint64_t t0 = globaltimer_ns();
      drain_wait(b_done_pv, 0, t0, tmo);
      for (int x = c; x < nv; ++x)
        drain_wait(b_vfull(x % C::VS), (x / C::VS) & 1, t0, tmo);
    }
  } else if (warp == 3 || (C::TWO_QK && warp == 1)) {
    if (lane == 0) {
      // ================= QK^T issuers: warp 3 the even groups, warp 1 the odd ones ====
      const int par = warp == 3 ? 0 : 1;
      constexpr int step = C::TWO_QK ? 2 : 1;
      constexpr uint32_t ID_FULL = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t ID_PAGE = idesc_bf16_f32(128, P, 0);  // a lone last page
      // descriptors of the tile bases; a 16-byte aligned offset below 256 KB adds to
      // the start-address field directly
      const uint64_t dq = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dk = smem_desc_sw128(sK, 16, 1024);
      bool ok = wait(b_q, 0);
      // Group g reads K ring slot g % KG (phase g / KG) and writes S buffer g % SBG,
      // which its previous user, group g - SBG, gave back on s_free[g % SBG][g % 2] in
      // phase (g - SBG) / (2 SBG).  Whether this thread's next group can go is tested
      // while the last MMAs of this one are still queued, and then it goes without a
      // wait.
      auto sfree_phase = [](int g) { return ((g - C::SBG) / (2 * C::SBG)) & 1; };
      bool next_ready = false;
      for (int g = par; ok && g < n_groups; g += step) {
        if (R > 0 && g >= *stop_g) break;  // past an early break: not issued
        const int ks = g % C::KG, sbuf = g % C::SBG;
        if (!next_ready) {
          if (wait_g(b_kfull(ks), (g / C::KG) & 1, g) != 1) break;
          if (g >= C::SBG && wait_g(b_sfree(sbuf, g & 1), sfree_phase(g), g) != 1) break;
        }
        tc_fence_after();
        const uint32_t id = (g * GP + GP <= n_list) ? ID_FULL : ID_PAGE;
        const uint64_t dks = dk + ((uint32_t)ks * C::KG_BYTES >> 4);
        const int g2 = g + step;
        next_ready = false;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          if (k == D / 16 - 2 && g2 < n_groups)
            next_ready = mbar_test_wait(b_kfull(g2 % C::KG), (g2 / C::KG) & 1) &&
                         (g2 < C::SBG || mbar_test_wait(b_sfree(g2 % C::SBG, g2 & 1),
                                                        sfree_phase(g2)));
          mma_bf16_ss(tmem + sbuf * 128, dq + (((k >> 2) * (C::QB * 128) + (k & 3) * 32) >> 4),
                      dks + (((k >> 2) * (GP * P * 128) + (k & 3) * 32) >> 4), id, k > 0 ? 1u : 0u);
        }
        mma_commit(b_kempty(ks));
        mma_commit(b_sfull(sbuf, g & 1));
      }
      // every MMA this thread issued completes before teardown frees TMEM
      const uint32_t bd = par == 0 ? b_done : b_done_odd;
      mma_commit(bd);
      const uint64_t t0 = globaltimer_ns();
      drain_wait(bd, 0, t0, tmo);
    }
  } else if (warp >= 4) {
    // ================= softmax: two warpgroups taking the groups in turn ========
    const int wg = (warp - 4) >> 2;      // groups g with g % 2 == wg
    const int q4 = warp & 3;             // TMEM lane quarter
    const int row = q4 * 32 + lane;
    const bool row_valid = row < prm.q_block;
    const int grow = row0 + row;
    const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
    const bool lead_warp = (q4 == 0);
    const bool leader = lead_warp && lane == 0;
    const float sl2 = prm.scale_log2, le = prm.log2_eps;
    float m_run = -INFINITY, m_ref = -INFINITY, l = 0.f;  // l: this warpgroup's share, base m_ref
    bool ok = true;     // OSK: collective within the warpgroup
    bool fail = false;  // this warp missed a wait after the vote; reported at the next vote
    // Page ids of list entries [fb, fb + 32) (lane l: entry fb + l) in pid_l and, in the
    // leading warp, their TMA coordinates in cz_l, loaded when the list reaches a new
    // block of 32 (loading the next block ahead was measured 4 % slower)
    int fb = -1, pid_l = 0, cz_l = 0;
    // page id (and, in the leading warp, TMA coordinate) of list entry j; j only grows
    auto fetch = [&](int j, int& cz) -> int {
      const int base = j & ~31;
      if (base != fb) {
        fb = base;
        const int jl = base + lane;
        pid_l = jl < n_list ? page_at(jl) : 0;
        if (lead_warp) cz_l = jl < n_list ? coord_of(pid_l) : 0;
      }
      cz = __shfl_sync(0xffffffffu, cz_l, j & 31);
      return __shfl_sync(0xffffffffu, pid_l, j & 31);
    };
    // row max of raw logits over the page at TMEM column col (key key0), 64 columns
    // at a time, causal mask on the diagonal page
    auto row_max = [&](uint32_t col, int key0) -> float {
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < P / 64; ++c) {
        uint32_t v[64];
        tmem_ld64(t_row + col + c * 64, v);
        const int k0 = key0 + c * 64;
        if (k0 + 63 > row0) {  // diagonal page (warp-uniform): causal mask
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (k0 + e > grow) v[e] = __float_as_uint(-INFINITY);
        }
        // 64 values to one with three-input maxima: eight running maxima take two
        // values at a time, then one more each, then three steps combine them
        float a[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(v[e]);
#pragma unroll
        for (int r = 8; r + 16 <= 64; r += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e)
            a[e] = fmax3f(a[e], __uint_as_float(v[r + e]), __uint_as_float(v[r + 8 + e]));
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] = fmaxf(a[e], __uint_as_float(v[56 + e]));
        mx = fmax3f(mx, fmax3f(a[0], a[1], a[2]), fmax3f(a[3], a[4], a[5]));
        mx = fmax3f(mx, a[6], a[7]);
      }
      return mx;
    };
    // leader: publish kept page c to the queue: its TMA coordinate (for the V
    // load), then its P column and last-of-group flag (for the PV issue)
    auto bounded_until = [&](volatile int* pos, int c) {
      if (c < C::KQ || *pos > c - C::KQ) return;
      const uint64_t t0 = globaltimer_ns();
      while (*pos <= c - C::KQ) {  // the entry's previous use has been read
        if (*abort_flag || timed_out(t0)) { give_up(); break; }
        __nanosleep(32);
      }
    };
    auto publish_v = [&](int c, int cz) {
      bounded_until(v_pos, c);
      kq[c % C::KQ].x = cz;
      __threadfence_block();
      *vq_count = c + 1;
    };
    uint8_t* slog = prm.skip_log ? prm.skip_log + (bh * prm.num_q_blocks + qb) * prm.k_cap
                                             : nullptr;
    // kept page c: P = exp2(s * scale - mb) (bf16 pairs) written over the page's first
    // P / 2 S columns, after the O rescale by alpha when this page moved the base
    auto kept_page = [&](uint32_t col, int key0, float mb, bool resc_any, float alpha,
                         int c) -> bool {
      if (resc_any) {
        // O holds the pages before c: wait for their last PV, rescale this warp's rows
        if (c > 0 && !wait_warp(b_pvdone((c - 1) % C::PD), ((c - 1) / C::PD) & 1)) return false;
        tc_fence_after();
#pragma unroll 1
        for (int k = 0; k < D / 16; ++k) {
          uint32_t r[16];
          tmem_ld16(t_row + C::COL_O + k * 16, r);
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st16(t_row + C::COL_O + k * 16, r);
        }
        tmem_st_wait();
        l *= alpha;
      }
      const bool diag = key0 + P - 1 > row0;
      const bool rlive = row_valid && mb != -INFINITY;
      const float nb2 = rlive ? -mb : 0.f;
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int k = 0; k < P / 64; ++k) {
        uint32_t cur[64];
        tmem_ld64(t_row + col + k * 64, cur);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int i0 = h2 * 32 + 2 * e, key = key0 + k * 64 + i0;
            float x0 = fmaf(__uint_as_float(cur[i0]), sl2, nb2);
            float x1 = fmaf(__uint_as_float(cur[i0 + 1]), sl2, nb2);
            if (!rlive || (diag && key > grow)) x0 = -INFINITY;
            if (!rlive || (diag && key + 1 > grow)) x1 = -INFINITY;
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            rs[e & 3] += p0 + p1;
            __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
            w[e] = *reinterpret_cast<uint32_t*>(&v2);
          }
          // S columns [k * 64, k * 64 + 64) are read: P pairs go to [k * 32, k * 32 + 32)
          tmem_st16(t_row + col + k * 32 + h2 * 16, w);
        }
      }
      l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_pfull(c % C::PF));
      return true;
    };
    // votes of this warpgroup's four warps for its iteration it
    auto vote_round = [&](int it, uint32_t bits) -> uint32_t {
      int* vt = const_cast<int*>(votes) + (wg * 2 + (it & 1)) * 4;
      if (lane == 0) vt[q4] = (int)bits;
      named_bar_sync(1 + wg, 128);  // orders the shared-memory exchange around it
      const int4 v = *reinterpret_cast<const int4*>(vt);
      return (uint32_t)(v.x | v.y | v.z | v.w);
    };
    // wait (lane 0 of each warp) until every warp of the other warpgroup has settled
    // group g (all groups before the next one of this warpgroup are then settled)
    // (1 done, 0 timeout or abort, 2 group g + 1 lies past an early break: group g may
    // never be settled, and g + 1 needs no state, all its pages being skipped)
    auto wait_settled = [&](int g) -> int {
      int okl = 1;
      if (lane == 0) {
        volatile int* o = settled + (wg ^ 1) * 4;
        auto done = [&]() { return min(min(o[0], o[1]), min(o[2], o[3])) >= g; };
        if (!done()) {
          const uint64_t t0 = globaltimer_ns();
          uint32_t spins = 0, nap = 32;
          while (!done()) {
            if (g + 1 >= *stop_g) { okl = 2; break; }
            if (*abort_flag) { okl = 0; break; }
            if ((++spins & 15u) == 0 && timed_out(t0)) { give_up(); okl = 0; break; }
            __nanosleep(nap);
            nap = min(nap * 2, 256u);
          }
        }
      }
      return __shfl_sync(0xffffffffu, okl, 0);
    };
    // this warp has settled group g (its state rows and queue entries are written)
    auto mark_settled = [&](int g) {
      __threadfence_block();
      __syncwarp();
      if (lane == 0) settled[wg * 4 + q4] = g;
    };
    // the first listed page is always kept: its V can go out before any vote
    if (wg == 0 && n_list > 0) {
      int cz0;
      fetch(0, cz0);
      if (leader) publish_v(0, cz0);
    }
    int rnd = 0;  // vote rounds of this warpgroup
    for (int g = wg; g < n_groups; g += 2) {
      const int j = g * GP;
      const int nb = min(GP, n_list - j);
      const int sb = g % C::SBG;
      int key0[GP], czp[GP];
#pragma unroll
      for (int t = 0; t < GP; ++t) {
        czp[t] = 0;
        key0[t] = t < nb ? fetch(j + t, czp[t]) * P : 0;
      }
      // ---- row maxima of the group's pages, read from TMEM.  One lane waits for S and
      // the named barrier brings the four warps along together (apart, each warp
      // waking on its own, the vote barrier waited for the last of them).
      // A group past an early break is not waited for (it may never be issued): the
      // warpgroup stops there.
      if (leader)
        s_ok[wg] = (R > 0 && g >= *stop_g) ? 2 : wait_g(b_sfull(sb, wg), (g / (2 * C::SBG)) & 1, g);
      named_bar_sync(1 + wg, 128);
      const int s_res = s_ok[wg];
      if (s_res == 2) break;
      const bool okw = !fail && s_res != 0;
      if (okw) tc_fence_after();
      // (one copy of the per-page code: the loop is not unrolled)
      float ml0 = -INFINITY, ml1 = -INFINITY;
#pragma unroll 1
      for (int t = 0; t < (okw ? nb : 0); ++t) {
        const float mr = row_max(sb * 128 + t * P, t == 0 ? key0[0] : key0[GP - 1]);
        if (t == 0) ml0 = mr;
        else ml1 = mr;
      }
      float mloc[GP];
      bool lv[GP];
#pragma unroll
      for (int t = 0; t < GP; ++t) {
        const float mr = row_valid ? (t == 0 ? ml0 : ml1) : -INFINITY;
        lv[t] = mr != -INFINITY;
        mloc[t] = lv[t] ? mr * sl2 : -INFINITY;
      }
      tc_fence_before();
      // votes of this group's pages against running max m: page 1 (2), page 2 after
      // page 1 kept (4), page 2 after page 1 skipped (8)
      auto vote_bits = [&](float m) -> uint32_t {
        const bool n0 = lv[0] && (m == -INFINITY || mloc[0] - m >= le);
        uint32_t bits = n0 ? 2u : 0u;
        if (GP == 2 && nb == 2) {
          const float mk = fmaxf(m, mloc[0]);
          const bool nk = lv[GP - 1] && (mk == -INFINITY || mloc[GP - 1] - mk >= le);
          const bool ns = lv[GP - 1] && (m == -INFINITY || mloc[GP - 1] - m >= le);
          bits |= (nk ? 4u : 0u) | (ns ? 8u : 0u);
        }
        return __reduce_or_sync(0xffffffffu, bits);  // the warp's votes
      };
      {
        const bool exact = j == 0;  // the first listed page is always kept
        // ---- first vote, against the running max this warpgroup last saw (a lower
        // bound of the current one: what it skips stays skipped)
        m_run = fmaxf(m_run, st_rows[row].x);
        uint32_t bits = okw ? 0u : 1u;
        if (okw && !exact) bits |= vote_bits(m_run);
        const uint32_t all = vote_round(rnd++, bits);
        if (all & 1u) { ok = false; break; }
        if (!exact && (all & 10u) == 0) {
          // every page of the group is skipped: settled without the other warpgroup
          if (leader) {
            if (slog)
              for (int t = 0; t < nb; ++t) slog[j + t] = 1;
            mbar_arrive(b_sfree(sb, wg ^ 1));
            // early break: once every group before this one is settled, the last kept
            // page is known; if the skipped run reaches R by the next group's first
            // page, every later group lies past the break
            if (R > 0) {
              volatile int* o = settled + (wg ^ 1) * 4;
              if (min(min(o[0], o[1]), min(o[2], o[3])) >= g - 1) {
                __threadfence_block();
                if ((g + 1) * GP - *kept_last - 1 >= R) atomicMin(const_cast<int*>(stop_g), g + 1);
              }
            }
          }
          // a skipped group writes no state rows or queue entries: nothing to order
          // before its settled mark (the last exact group's writes were fenced)
          __syncwarp();
          if (lane == 0) settled[wg * 4 + q4] = g;
          continue;
        }
      }
      // ---- exact path: the groups before this one are settled; take their state
      const int wsr = !okw ? 0 : (g == 0 ? 1 : wait_settled(g - 1));
      const bool oks = wsr == 1;
      if (oks) {
        __threadfence_block();
        const float sr = st_rows[row].x, sf = st_rows[row].y;
        if (sf != m_ref) {  // the base only moves up: bring this warpgroup's l along
          if (m_ref != -INFINITY) l *= ex2_approx(m_ref - sf);
          m_ref = sf;
        }
        m_run = sr;
      }
      // kept pages before this group: every earlier queue entry is published, and
      // the count is read before the vote barrier, ahead of this group's publishing
      const int c0 = *kq_count;
      // early break: list position of the last kept page before this group; a page with
      // R skipped pages right before it, and every page after it, is skipped unvisited
      const int kl = (R > 0 && oks) ? *kept_last : -1;
      bool keep[GP];
      {
        // bit 16: page j lies past the break (said by every warp that knows it)
        uint32_t bits = oks ? vote_bits(m_run) : (wsr == 2 ? 16u : 1u);
        if (oks && R > 0 && j - kl - 1 >= R) bits |= 16u;
        const uint32_t all = vote_round(rnd++, bits);
        if (all & 1u) { ok = false; break; }
        const bool past0 = (all & 16u) != 0;
        keep[0] = !past0 && ((j == 0) || (all & 2u));
        if (GP == 2) {
          const bool past1 = past0 || (R > 0 && !keep[0] && j - kl >= R);
          keep[GP - 1] = !past1 && nb == 2 && (keep[0] ? (all & 4u) != 0 : (all & 8u) != 0);
        }
      }
      // ---- state after this group's decisions: running max, and the exponent base
      // (with the O rescale factor) of each kept page
      float mb[GP], alpha[GP];
      bool rany[GP];
      int nk = 0, lastk = -1;
#pragma unroll
      for (int t = 0; t < GP; ++t) {
        mb[t] = m_ref;
        alpha[t] = 1.f;
        rany[t] = false;
        if (t < nb && keep[t]) {
          const float m_new = fmaxf(m_run, mloc[t]);
          m_run = m_new;
          const bool resc = (m_ref != -INFINITY) && (m_new > m_ref + kRescaleLog2);
          rany[t] = __any_sync(0xffffffffu, resc);
          // (the exponential only in the rare warp that rescales: the special-function
          // unit is busy with the other warpgroup's P)
          if (rany[t] && resc) alpha[t] = ex2_approx(m_ref - m_new);
          if (m_new != -INFINITY && (m_ref == -INFINITY || resc)) m_ref = m_new;
          mb[t] = m_ref;
          ++nk;
          lastk = t;
        }
      }
      if (nk > 0) {
        st_rows[row].x = m_run;
        st_rows[row].y = m_ref;
      }
      if (leader) {
        int c = c0;
        bool new_v = false;
#pragma unroll
        for (int t = 0; t < GP; ++t)
          if (t < nb) {
            if (slog) slog[j + t] = keep[t] ? 0 : 1;
            if (keep[t]) {
              // the entry's coordinate (for the V load; page 0's went out before any
              // vote) and P location (for the PV issue), once its previous use is read
              if (j + t > 0) {
                bounded_until(v_pos, c);
                kq[c % C::KQ].x = czp[t];
                new_v = true;
              }
              bounded_until(pv_pos, c);
              kq[c % C::KQ].y = (sb * 128 + t * P) | ((t == lastk ? 1 : 0) << 15) | (wg << 16);
              ++c;
            }
          }
        if (c > c0) {  // entries before counts
          __threadfence_block();
          if (new_v) *vq_count = c;
          *kq_count = c;
        }
        if (nk == 0) mbar_arrive(b_sfree(sb, wg ^ 1));  // nothing kept: the S buffer goes back now
        if (R > 0 && oks) {  // early break: the last kept page, and whether the rest is past it
          const int kl2 = nk > 0 ? j + lastk : kl;
          if (nk > 0) *kept_last = kl2;
          if ((g + 1) * GP - kl2 - 1 >= R) atomicMin(const_cast<int*>(stop_g), g + 1);
        }
      }
      mark_settled(g);
      // ---- P of the kept pages; their PV follows in list order
      int c = c0;
#pragma unroll 1
      for (int t = 0; t < nb; ++t) {
        const bool k1 = t > 0;  // (scalar selects keep one copy of the page code)
        if (!(k1 ? keep[GP - 1] : keep[0])) continue;
        if (!fail && !kept_page(sb * 128 + t * P, k1 ? key0[GP - 1] : key0[0],
                                k1 ? mb[GP - 1] : mb[0], k1 ? rany[GP - 1] : rany[0],
                                k1 ? alpha[GP - 1] : alpha[0], c))
          fail = true;
        ++c;
      }
    }
    if (leader) {  // the second warpgroup to finish closes the queue
      __threadfence_block();
      if (atomicAdd(wg_done, 1) == 1) {
        *kq_final = *kq_count;
        // pages of groups past an early break that no warpgroup reached: skipped
        if (slog && R > 0)
          for (int p = *stop_g * GP; p < n_list; ++p) slog[p] = 1;
      }
    }
    // ---- epilogue: both warpgroups' row sums to one base, O / l -> bf16, LSE
    fin_rows[wg * 128 + row].x = l;
    fin_rows[wg * 128 + row].y = m_ref;
    __threadfence_block();
    named_bar_sync(3, 256);
    const float ol = fin_rows[(wg ^ 1) * 128 + row].x, om = fin_rows[(wg ^ 1) * 128 + row].y;
    const float M = fmaxf(m_ref, om);
    float lt = 0.f;
    if (m_ref != -INFINITY) lt += l * ex2_approx(m_ref - M);
    if (om != -INFINITY) lt += ol * ex2_approx(om - M);
    const int cfin = *kq_count;
    int hv = 0;
    if (lane == 0) hv = (*abort_flag == 0 && cfin > 0) ? 1 : 0;
    bool have = __shfl_sync(0xffffffffu, hv, 0) != 0;
    if (have) have = wait_warp(b_pvdone((cfin - 1) % C::PD), ((cfin - 1) / C::PD) & 1);
    tc_fence_after();
    const float inv = (have && lt > 0.f) ? 1.f / lt : 0.f;
    constexpr int HD = D / 2;  // each warpgroup writes half of the columns
    __nv_bfloat16* orow = prm.out + (bh * prm.seq_len + grow) * D + wg * HD;
#pragma unroll 1
    for (int k = 0; k < HD / 32; ++k) {
      uint32_t r[32];
      if (have) {
        tmem_ld32(t_row + C::COL_O + wg * HD + k * 32, r);
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
    if (wg == 0 && row_valid && prm.lse)
      prm.lse[bh * prm.seq_len + grow] =
          (have && lt > 0.f) ? (M + log2f(lt)) * 0.69314718055994531f : -INFINITY;
    if (wg == 0 && leader && prm.computed) prm.computed[bh * prm.num_q_blocks + qb] = cfin;
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (R > 0 && tid == 0) {
    // After an early break some K copies may never have been consumed: wait for the last
    // copy into every ring slot.  Slot s holds groups s, s + KG, ... in order, each
    // loaded only after the one before it was read, so its last copy is the largest
    // loaded group g = s (mod KG), phase g / KG; the producers loaded prefixes of their
    // groups (group g by warp g % NPROD).
    const uint64_t t0 = globaltimer_ns();
    for (int s = 0; s < C::KG; ++s) {
      int best = -1;
      for (int kp = 0; kp < C::NPROD; ++kp)
        for (int g = k_last[kp]; g >= 0 && g > k_last[kp] - C::NPROD * C::KG; g -= C::NPROD)
          if (g % C::KG == s) {
            best = max(best, g);
            break;
          }
      if (best >= 0)
        drain_wait(b_kfull(s), (best / C::KG) & 1, t0, tmo);
    }
  }
  if (warp == 3) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace cosa
