// Dense causal attention on the sm_100a tensor cores: the comparison point the
// sparse path is measured against (every causal key of every query, the softmax
// of gist.science/pt "CoSA" technical summary §2.3 with nothing skipped).
//
// One CTA (384 threads) per (b, h_q, pair of 128-row query tiles).  Both tiles
// read the same 128-key K/V blocks, so each block crosses from L2 into shared
// memory once for 256 query rows.  Each tile has its own S (128 columns) and O
// (D columns) in TMEM; P (bf16 pairs) is written over the first 64 columns of its
// tile's S and read from there by the PV MMA.
//   warp 0   Q and K loads (TMA through the page table, no multicast)
//   warp 1   MMA issue (one thread), in the order
//              QK0(0) QK1(0) | PV0(0) QK0(1) | PV1(0) QK1(1) | PV0(1) QK0(2) | ...
//            so that while one tile's softmax runs the tensor core works on the
//            other tile.  tcgen05.mma operations of one thread execute in issue
//            order, so QKi(j+1) overwrites Si only after PVi(j) has read Pi(j).
//   warp 2   V loads
//   warp 3   TMEM allocation
//   warps 4-7 / 8-11  softmax of tile 0 / tile 1, one query row per thread (its
//            TMEM lane).  Row max over the block, then P = exp2(s * scale - m_ref);
//            the exponent base m_ref moves only when the row max passes it by
//            more than 2^8 (O and l are then rescaled in TMEM; the commit that
//            reports Si full also covers PVi(j-1), so O is at rest), which keeps
//            P <= 256.  S is read twice, all 128 columns in one load for the max and
//            32 at a time (the next 32 loading meanwhile) for P; the causal mask runs
//            on the diagonal block only.  The two hand-offs of the cycle (S full to
//            the softmax, P full to the MMA thread) are polled without suspending.
// Every wait is bounded: on timeout the CTA records COSA_ERR_TIMEOUT in the status
// word, drains what it issued, frees TMEM and exits.
#pragma once

#include <type_traits>

#include "attn_tc.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace cosa {

template <int D, int P>
struct DenseCfg {
  static constexpr int QB = 128;                   // rows per tile
  static constexpr int KB = 128;                   // keys per block
  static constexpr int NT = 384;
  static constexpr uint32_t Q_BYTES = QB * D * 2;  // one tile
  static constexpr uint32_t BLK_BYTES = KB * D * 2;  // one K or V block
  static constexpr uint32_t PAGE_BYTES = P * D * 2;
  static constexpr int KS = (D == 128) ? 3 : 4;    // K ring slots (blocks)
  static constexpr int VS = (D == 128) ? 2 : 4;    // V ring slots (blocks)
  static constexpr uint32_t OFF_Q = 0;             // two tiles
  static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KS * BLK_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + VS * BLK_BYTES;
  // q, k_full/empty, v_full/empty, s_full[2], p_full[2], o_full[2], done
  static constexpr int NBAR = 1 + 2 * KS + 2 * VS + 6 + 1;
  static constexpr uint32_t OFF_MISC = (OFF_BAR + NBAR * 8 + 15) & ~15u;  // TMEM address, abort
  static constexpr uint32_t SMEM = OFF_MISC + 16;
  static constexpr uint32_t SMEM_ALLOC = SMEM + 1024;  // 1024-byte alignment slack
  static constexpr int TMEM_COLS = 512;
  static constexpr int COL_O = 256;                // O of tile i at COL_O + i * D
  static constexpr float kRescale = 8.0f;          // log2 slack of the exponent base
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory budget");
  static_assert(COL_O + 2 * D <= TMEM_COLS, "TMEM budget");
  static_assert(KB % P == 0 && BLK_BYTES % 1024 == 0, "blocks of whole pages, 1024-byte aligned");
};

template <int D, int P>
__global__ void __launch_bounds__(384, 1)
    attn_dense_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const TcParams prm) {
  using C = DenseCfg<D, P>;
  using namespace tc;
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
  auto b_pfull = [&](int i) { return bar + 8u * (3 + 2 * C::KS + 2 * C::VS + i); };
  auto b_ofull = [&](int i) { return bar + 8u * (5 + 2 * C::KS + 2 * C::VS + i); };
  const uint32_t b_done = bar + 8u * (C::NBAR - 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sg + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sg + C::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (__syncthreads_or(*(volatile int*)&g_status == COSA_ERR_TIMEOUT)) return;

  // ---- work decode: KV-head major, heaviest tile pairs first, G heads fastest
  const int N = prm.seq_len, G = prm.group;
  const int npairs = (N + 2 * C::QB - 1) / (2 * C::QB);
  const int per_kv = G * npairs;
  const int z = blockIdx.x / per_kv;
  const int rem = blockIdx.x % per_kv;
  const int tp = npairs - 1 - rem / G;
  const int hk = z % prm.num_kv_heads;
  const int b = z / prm.num_kv_heads;
  const int h = hk * G + rem % G;
  const long long bh = (long long)b * prm.num_q_heads + h;
  // tile i: first row, rows inside the sequence, key blocks up to the diagonal one
  const int r00 = 2 * tp * C::QB, r01 = r00 + C::QB;
  const int rows0 = max(0, min(C::QB, N - r00)), rows1 = max(0, min(C::QB, N - r01));
  const int nbt0 = rows0 > 0 ? r00 / C::KB + 1 : 0, nbt1 = rows1 > 0 ? r01 / C::KB + 1 : 0;
  auto r0 = [&](int i) { return i ? r01 : r00; };
  auto rows = [&](int i) { return i ? rows1 : rows0; };
  auto nbt = [&](int i) { return i ? nbt1 : nbt0; };
  const int nb = max(nbt0, nbt1);
  const int32_t* ptab = prm.page_table + (long long)b * prm.pages_per_seq;
  // keys in block j (the last block of an odd number of 64-key pages holds 64)
  auto blk_keys = [&](int j) { return min(C::KB, N - j * C::KB); };

  // ---- setup
  if (tid == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < C::KS; ++s) { mbar_init(b_kfull(s), 1); mbar_init(b_kempty(s), 1); }
    for (int s = 0; s < C::VS; ++s) { mbar_init(b_vfull(s), 1); mbar_init(b_vempty(s), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_sfull(i), 1);
      mbar_init(b_pfull(i), 4);
      mbar_init(b_ofull(i), 1);
    }
    mbar_init(b_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 3) {
    tmem_alloc(sb0 + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  // a tile with 64 rows (N odd in 64-row halves) gets zeros in its second half;
  // the TMA loads only whole 64-row halves inside the sequence
  if (warp >= 4) {
    const int i = (warp - 4) >> 2;
    if (rows(i) > 0 && rows(i) < C::QB) {
      for (int x = tid & 127; x < (D / 64) * 64 * 8; x += 128) {
        const int chunk = x & 7, r = 64 + ((x >> 3) & 63), kb = x >> 9;
        st_shared_v4(sQ + i * C::Q_BYTES + kb * (C::QB * 128) + r * 128 + chunk * 16, 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
    }
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
    while (!mbar_try_wait(bar_addr, parity)) {
      if (*abort_flag) return false;
      if (*(volatile int*)&g_status == COSA_ERR_TIMEOUT || globaltimer_ns() - t0 > tmo) {
        give_up();
        return false;
      }
    }
    return true;
  };
  auto wait_warp = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    int okl = 1;
    if (lane == 0) okl = wait(bar_addr, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, okl, 0) != 0;
  };
  // the same without suspending: for the hand-offs on the softmax / MMA cycle
  auto wait_hot = [&](uint32_t bar_addr, uint32_t parity) -> bool {
    if (mbar_test_wait(bar_addr, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t n = 0;
    while (!mbar_test_wait(bar_addr, parity)) {
      if ((++n & 255u) == 0) {
        if (*abort_flag) return false;
        if (*(volatile int*)&g_status == COSA_ERR_TIMEOUT || globaltimer_ns() - t0 > tmo) {
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
  // TMA loads of block j into ring slot s (1 or 2 pages)
  auto load_block = [&](const CUtensorMap* tm, uint32_t dst, uint32_t full_bar, int j) {
    const int np = blk_keys(j) / P;
    mbar_arrive_expect_tx(full_bar, (uint32_t)np * C::PAGE_BYTES);
    for (int pg = 0; pg < np; ++pg) {
      const int cz = __ldg(ptab + j * (C::KB / P) + pg) * prm.num_kv_heads + hk;
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_3d(dst + kb * (C::KB * 128) + pg * (P * 128), tm, full_bar, kb * 64, 0, cz);
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      // ================= Q (whole 64-row halves inside the sequence) and K ========
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      uint32_t qbytes = 0;
      for (int i = 0; i < 2; ++i)
        for (int hf = 0; hf < 2; ++hf)
          if (rows(i) > 64 * hf) qbytes += (D / 64) * 64 * 128;
      mbar_arrive_expect_tx(b_q, qbytes);
      for (int i = 0; i < 2; ++i)
        for (int hf = 0; hf < 2; ++hf)
          if (rows(i) > 64 * hf) {
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_3d(sQ + i * C::Q_BYTES + kb * (C::QB * 128) + hf * (64 * 128), &tm_q, b_q,
                          kb * 64, r0(i) + 64 * hf, (int)bh);
          }
      int j = 0;
      for (; j < nb; ++j) {
        const int s = j % C::KS;
        if (j >= C::KS && !wait(b_kempty(s), ((j / C::KS) - 1) & 1)) break;
        load_block(&tm_k, sK + s * C::BLK_BYTES, b_kfull(s), j);
      }
      // loads never consumed (abort only) land before the CTA leaves
      const uint64_t t0 = globaltimer_ns();
      drain_wait(b_q, 0, t0, tmo);
      for (int x = max(0, j - C::KS); x < j; ++x)
        drain_wait(b_kfull(x % C::KS), (x / C::KS) & 1, t0, tmo);
    }
  } else if (warp == 2) {
    if (lane == 0) {
      // ================= V ========================================================
      prefetch_tmap(&tm_v);
      int j = 0;
      for (; j < nb; ++j) {
        const int s = j % C::VS;
        if (j >= C::VS && !wait(b_vempty(s), ((j / C::VS) - 1) & 1)) break;
        load_block(&tm_v, sV + s * C::BLK_BYTES, b_vfull(s), j);
      }
      const uint64_t t0 = globaltimer_ns();
      for (int x = max(0, j - C::VS); x < j; ++x)
        drain_wait(b_vfull(x % C::VS), (x / C::VS) & 1, t0, tmo);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================= MMA issue ================================================
      constexpr uint32_t ID_QK = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t ID_QK64 = idesc_bf16_f32(128, 64, 0);  // a 64-key last block
      constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, 1);
      // tile bases; a 16-byte aligned offset below 256 KB adds to the start-address field
      const uint64_t dq = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dk = smem_desc_sw128(sK, 16, 1024);
      const uint64_t dv = smem_desc_sw128(sV, C::KB * 128, 1024);
      // S_i = Q_i K_j^T
      auto qk = [&](int i, int j) {
        const uint32_t id = blk_keys(j) == C::KB ? ID_QK : ID_QK64;
        const uint64_t dqi = dq + ((uint32_t)i * C::Q_BYTES >> 4);
        const uint64_t dks = dk + ((uint32_t)(j % C::KS) * C::BLK_BYTES >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_ss(tmem + i * 128, dqi + (((k >> 2) * (C::QB * 128) + (k & 3) * 32) >> 4),
                      dks + (((k >> 2) * (C::KB * 128) + (k & 3) * 32) >> 4), id, k > 0 ? 1u : 0u);
        mma_commit(b_sfull(i));
      };
      // O_i += P_i V_j, P_i from TMEM (16 keys per step = 8 columns)
      auto pv = [&](int i, int j) {
        const uint64_t dvs = dv + ((uint32_t)(j % C::VS) * C::BLK_BYTES >> 4);
        const int nk = blk_keys(j) / 16;
        for (int k = 0; k < nk; ++k)
          mma_bf16_ts(tmem + C::COL_O + i * D, tmem + i * 128 + k * 8, dvs + ((k * 16 * 128) >> 4),
                      ID_PV, (j > 0 || k > 0) ? 1u : 0u);
      };
      bool ok = wait(b_q, 0) && wait(b_kfull(0), 0);
      if (ok) {
        tc_fence_after();
        for (int i = 0; i < 2; ++i)
          if (nbt(i) > 0) qk(i, 0);
        mma_commit(b_kempty(0));
      }
      for (int j = 0; ok && j < nb; ++j) {
        const int vs = j % C::VS;
        if (!wait(b_vfull(vs), (j / C::VS) & 1)) break;
        bool k_next = false;  // K of block j + 1 is in shared memory
        for (int i = 0; i < 2 && ok; ++i) {
          if (j >= nbt(i)) continue;
          if (!wait_hot(b_pfull(i), j & 1)) { ok = false; break; }
          tc_fence_after();
          pv(i, j);
          if (j + 1 < nbt(i)) {
            if (!k_next) {
              if (!wait(b_kfull((j + 1) % C::KS), ((j + 1) / C::KS) & 1)) { ok = false; break; }
              tc_fence_after();
              k_next = true;
            }
            qk(i, j + 1);
            if (i == 1 || j + 1 >= nbt(1)) mma_commit(b_kempty((j + 1) % C::KS));  // last reader
          } else {
            mma_commit(b_ofull(i));
          }
        }
        if (!ok) break;
        mma_commit(b_vempty(vs));
      }
      // every issued MMA completes before teardown frees TMEM
      mma_commit(b_done);
      const uint64_t t0 = globaltimer_ns();
      drain_wait(b_done, 0, t0, tmo);
    }
  } else if (warp >= 4) {
    // ================= softmax of tile i, one row per thread ========================
    const int i = (warp - 4) >> 2, q4 = warp & 3, row = q4 * 32 + lane;
    const int grow = r0(i) + row;
    const bool row_valid = row < rows(i);
    const uint32_t t_row = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t t_s = t_row + i * 128, t_o = t_row + C::COL_O + i * D;
    const float sl2 = prm.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nbt(i); ++j) {
      if (!wait_warp_hot(b_sfull(i), j & 1)) { ok = false; break; }
      tc_fence_after();
      const bool diag = (j == nbt(i) - 1);  // the only block with keys past some row
      const int key0 = j * C::KB;
      // S is read twice: all 128 columns at once for the row max (one load
      // latency), then 32 at a time with the next 32 loading meanwhile for P.
      // Keys past the row are masked on the diagonal block only: the other blocks
      // run the same code without the mask.
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      auto block = [&](auto mask_tag) {
        constexpr bool MASK = decltype(mask_tag)::value;
        auto val = [&](uint32_t v, int key) {
          return (MASK && key > grow) ? -INFINITY : __uint_as_float(v);
        };
        // ---- row max of the raw logits
        float m_loc;
        {
          uint32_t sa[64], sb[64];
          tmem_ld64_async(t_s, sa);
          tmem_ld64_async(t_s + 64, sb);
          tmem_ld_wait64x2(sa, sb);
          float a[8];
#pragma unroll
          for (int e = 0; e < 64; ++e)
            a[e & 7] = e < 8 ? val(sa[e], key0 + e) : fmaxf(a[e & 7], val(sa[e], key0 + e));
#pragma unroll
          for (int e = 0; e < 64; ++e) a[e & 7] = fmaxf(a[e & 7], val(sb[e], key0 + 64 + e));
#pragma unroll
          for (int w = 4; w > 0; w >>= 1)
#pragma unroll
            for (int e = 0; e < w; ++e) a[e] = fmaxf(a[e], a[e + w]);
          // key0 <= grow on the diagonal block: finite for rows in the sequence
          m_loc = a[0] * sl2;
        }
        const bool resc = m_loc > m_ref + C::kRescale;  // true on the first block
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
          const float alpha = resc ? ex2_approx(m_ref - m_loc) : 1.f;
#pragma unroll 1
          for (int k = 0; k < D / 32; ++k) {
            uint32_t r[32];
            tmem_ld32(t_o + k * 32, r);
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(t_o + k * 32, r);
          }
          tmem_st_wait();
          l *= alpha;
        }
        if (resc) m_ref = m_loc;
        // ---- P = exp2(s * scale - m_ref) as bf16 pairs: S columns [32c, 32c + 32)
        // give P columns [16c, 16c + 16), inside S columns already read
        const float nb2 = -m_ref;
        uint32_t va[32], vb[32], w[16];
        tmem_ld32_async(t_s, va);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t* cur = (c & 1) ? vb : va;
          uint32_t* nxt = (c & 1) ? va : vb;
          tmem_ld_wait32(cur);
          if (c < 3) tmem_ld32_async(t_s + (c + 1) * 32, nxt);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int key = key0 + c * 32 + 2 * e;
            const float x0 = fmaf(val(cur[2 * e], key), sl2, nb2);
            const float x1 = fmaf(val(cur[2 * e + 1], key + 1), sl2, nb2);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            rs[e & 3] += p0;
            rs[(e + 2) & 3] += p1;
            __nv_bfloat162 v2 = __floats2bfloat162_rn(p0, p1);
            w[e] = *reinterpret_cast<uint32_t*>(&v2);
          }
          tmem_st16(t_s + c * 16, w);
        }
      };
      if (diag) block(std::true_type{});
      else block(std::false_type{});
      l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_pfull(i));
    }
    // ---- epilogue: O / l -> bf16, LSE (natural log)
    if (nbt(i) > 0) {
      const bool have = ok && wait_warp(b_ofull(i), 0);
      tc_fence_after();
      const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* orow = prm.out + (bh * N + grow) * D;
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
        prm.lse[bh * N + grow] = (have && l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
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
