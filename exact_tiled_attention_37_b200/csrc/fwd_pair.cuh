// Forward attention with 2-CTA tensor-core products (tcgen05 .cta_group::2),
// the "2-CTA MMA" the "FlashAttention-4: Algorithm and Kernel Pipelining for
// Blackwell GPUs" finding on the FlashAttention entity page lists among the
// Blackwell techniques.
//
// fwd_pair_kernel: a cluster of two CTAs (ranks 0 and 1, on the two SMs of
// one TPC) owns two 128-row query tiles that read the same keys -- two query
// heads of one GQA group at the same query tile, or (without such a group)
// two adjacent query tiles of one head.  Each CTA keeps the single-tile
// forward's structure (64-row key tiles, S0 | S1 | O in 256 TMEM columns, two
// CTAs per SM, a softmax warpgroup that owns one row per thread), but the
// products are issued once for the pair by rank 0:
//
//   S  = [Q_0; Q_1] K_j^T   M = 256, N = 64 keys: rank r supplies its Q tile
//                            (A rows) and key rows 64 j + 32 r .. + 31 (B)
//   O += [P_0; P_1] V_j     M = 256, N = D: A = each CTA's P in its own TMEM,
//                            rank r supplies the D columns [64 r, 64 r + 64)
//                            of V_j's 64 rows (B)
//
// so each CTA loads half of every K and V tile (8 KB instead of 16 KB at
// D = 128) and each SM reads 5 KB of shared-memory operands per K = 16 step
// of S instead of 6 KB (an N = 64 product of one CTA is bound by that read:
// 48 cycles instead of 32).  Accumulators stay per CTA: rows of S and O of
// rank r are in rank r's tensor memory, lane = query row.
//
// Barriers: TMA loads of both CTAs report their bytes to rank 0's full
// barriers; rank 0's commits reach both CTAs' S / stage-free / O barriers
// (one instruction each); both softmax warpgroups arrive on rank 0's P
// barriers (8 warps).  The ring holds NS / 2 stages of one K half and one V
// half; a stage frees when its tile's P V product completes, which is also
// what the correction waits for, so each key tile costs two commits (S and
// stage-free): a commit occupies the tensor pipe about as long as a short
// product.
// Every wait is bounded (PairWaiter); both CTAs meet at a cluster barrier
// before tensor memory is released, so neither leaves while the other's
// products may still touch its memory.
#pragma once

#include "fwd.cuh"
#include "pair.cuh"

// 1: a commit both CTAs' barriers must see is one instruction with a two-CTA
// mask; 0: one instruction per CTA (kept for comparison).
#ifndef ETA_PAIR_COMMIT_MASK
#define ETA_PAIR_COMMIT_MASK 1
#endif

namespace eta {

template <int D, int BC, int NS>
struct PairCfg {
  static constexpr int ROWB = D * 2;               // bf16 rows
  static constexpr int NCHUNK = ROWB / 128;        // 128-byte chunks per row
  static constexpr int QCHUNK = 128 * 128;         // chunk of the 128-row Q tile
  static constexpr int QTILE = 128 * ROWB;
  static constexpr int KROWS = BC / 2;             // key rows of a K tile this CTA loads
  static constexpr int KCHUNK = KROWS * 128;       // chunk of this CTA's K half
  static constexpr int KHALF = KROWS * ROWB;
  static constexpr int VCH = NCHUNK / 2;           // D chunks of a V tile this CTA loads
  static constexpr int VHALF = BC * 128 * VCH;
  static constexpr int SLOT = KHALF > VHALF ? KHALF : VHALF;
  static constexpr int QK_STEPS = ROWB / 32;
  static constexpr int PV_STEPS = BC / 16;
  static constexpr int S_COL = 0, O_COL = 2 * BC, TMEM_COLS = 256;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_KV = QTILE;
  static constexpr int NSTG = NS / 2;             // stages: K half + V half of one key tile
  static constexpr int SMEM_BAR = SMEM_KV + NS * SLOT;
  // q_full, kv_full[NS] (rank 0's count both halves; K in slot 2 s, V in
  // 2 s + 1 of stage s), stage_free[NSTG] (P V of the stage's tile done),
  // s_full[2], p_full[2] (rank 0's: 8 warps), o_full, done
  static constexpr int BAR_Q = 0, BAR_KVF = 1, BAR_STE = 1 + NS, BAR_S = 1 + NS + NSTG,
                       BAR_P = 3 + NS + NSTG, BAR_O = 5 + NS + NSTG, BAR_DONE = 6 + NS + NSTG,
                       NBAR = 7 + NS + NSTG;
  static constexpr int SMEM_MISC = SMEM_BAR + 8 * NBAR;
  static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;
  static constexpr int THREADS = 256;
  static_assert(D == 128, "the V half is one 128-byte chunk of each row");
  static_assert(NS % 2 == 0, "K and V slots in pairs");
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
  static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
};

// heads_paired != 0: the pair is query heads (2i, 2i + 1) of one GQA group at
// query tile blockIdx.z (grid Hq x B x tiles); otherwise query tiles
// (2t, 2t + 1) of head blockIdx.x / 2 (grid 2 Hq x B x ceil(tiles / 2)).
// Longest causal work first in both.
template <int D, int BC, int NS>
__global__ void __launch_bounds__(256, 2)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const FwdParams p,
                    const int heads_paired) {
  using C = PairCfg<D, BC, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::SMEM_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC + 4);

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = (p.N + 127) / 128;
  int h, qb, qb_other;
  if (heads_paired) {
    h = blockIdx.x;
    qb = T - 1 - static_cast<int>(blockIdx.z);
    qb_other = qb;
  } else {
    h = blockIdx.x >> 1;
    const int pp = static_cast<int>(gridDim.z) - 1 - static_cast<int>(blockIdx.z);
    qb = 2 * pp + static_cast<int>(rank);
    qb_other = 2 * pp + static_cast<int>(rank ^ 1u);
  }
  const int b = blockIdx.y;
  const int hk = h / p.group;
  const int q0 = qb * 128;
  // both CTAs run the union of their key-tile ranges (tiles outside a row's
  // window are masked for it); both compute the same union
  const int2 ka = key_tiles(q0, p.N, p.wl, p.wr, BC);
  const int2 kb = key_tiles(qb_other * 128, p.N, p.wl, p.wr, BC);
  int j0 = ka.x, j1 = ka.y;
  if (kb.x < kb.y) {
    if (j0 < j1) {
      j0 = min(j0, kb.x);
      j1 = max(j1, kb.y);
    } else {
      j0 = kb.x;
      j1 = kb.y;
    }
  }
  const int n = max(0, j1 - j0);

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::BAR_Q), 1);
    for (int s = 0; s < NS; ++s) mbar_init(BAR(C::BAR_KVF + s), 1);
    for (int s = 0; s < C::NSTG; ++s) mbar_init(BAR(C::BAR_STE + s), 1);
    mbar_init(BAR(C::BAR_S + 0), 1);
    mbar_init(BAR(C::BAR_S + 1), 1);
    mbar_init(BAR(C::BAR_P + 0), 8);
    mbar_init(BAR(C::BAR_P + 1), 8);
    mbar_init(BAR(C::BAR_O), 1);
    mbar_init(BAR(C::BAR_DONE), 1);
    *abort_flag = 0u;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 5) {
    tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barrier inits and tensor memory of both CTAs are in place
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const PairWaiter W{abort_flag, p.status, p.wait_limit_ns};
  const uint32_t lbar0 = mapa_shared(bar0, 0u);         // rank 0's barriers
  const uint32_t pbar0 = mapa_shared(bar0, rank ^ 1u);  // the other CTA's barriers
  const uint32_t obar0 = mapa_shared(bar0, rank);       // this CTA's, as cluster addresses
  auto LBAR = [&](int i) -> uint32_t { return lbar0 + 8u * static_cast<uint32_t>(i); };

  if (warp < 4) {
    // ---------------------------------------- softmax, correction, epilogue
    const int r = threadIdx.x & 127;
    const int qrow = q0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t o_addr = tmem + lane_base + C::O_COL;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int u = 0; u < n; ++u) {
      const int j = j0 + u;
      const int buf = u & 1;
      const uint32_t s_addr = tmem + lane_base + C::S_COL + BC * buf;
      if (!W.wait_warp(BAR(C::BAR_S + buf), (u >> 1) & 1, 60)) { ok = false; break; }
      tc_fence_after();
      const int2 cw = col_window(BC * j, qrow, p.N, p.wl, p.wr);
      bool rescaled = false;
      float alpha = 1.f;
      if (__all_sync(0xffffffffu, cw.y <= 0 || cw.x >= BC || cw.x >= cw.y)) {
        // no row of this warp sees a key of the tile (the other CTA's tile
        // reaches further): P = 0 and the row state stays
        uint32_t z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
        for (int c = 0; c < BC / 64; ++c) tmem_st32(s_addr + 32 * c, z);
      } else {
        float s[BC];
        tmem_load_row<BC>(s_addr, s);
        apply_mask<BC>(s, cw);
        rescaled = online_softmax_step<BC, kSoftExp8>(s, p.c, m, l, alpha);
        tmem_store_p<BC, false>(s_addr, s);
      }
      if (rescaled && u > 0) {
        // O must hold every P V product up to tile u-1 before it is rescaled:
        // tile u-1's stage frees when its product completes
        const int pu = u - 1;
        if (!W.wait_warp(BAR(C::BAR_STE + pu % C::NSTG), (pu / C::NSTG) & 1, 61)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_scale_row<D>(o_addr, alpha);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(LBAR(C::BAR_P + (u & 1)));
    }
    if (ok && n == 0) {
      store_empty_row<__nv_bfloat16, D>(p, b, h, qrow);
    } else if (ok && W.wait_warp(BAR(C::BAR_O), 0, 62)) {
      tc_fence_after();
      // O / l through TMA stores staged in this warp's rows of Q's first
      // chunk (every product reading Q is complete)
      uint8_t* stage = smem + C::SMEM_Q + warp * 32 * 128;
      tmem_rows_tma_store<D>(o_addr, stage, &tm_o, 0, q0 + warp * 32, h, b,
                             l > 0.f ? p.o_mul / l : 0.f);
      if (qrow < p.N)
        p.lse[(static_cast<long long>(b) * p.Hq + h) * p.N + qrow] =
            l > 0.f ? m * p.scale + logf(l) : -INFINITY;
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
    }
  } else if (warp == 4) {
    // ---------------------------------------- TMA producer of this CTA's halves
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (leader) mbar_expect_tx(BAR(C::BAR_Q), 2 * C::QTILE);
      tma_load_5d_pair(sbase + C::SMEM_Q, &tm_q, LBAR(C::BAR_Q), 0, q0, 0, h, b);
      int issued = 0;  // key tiles whose stage was claimed
      for (int u = 0; u < n && !W.aborted(); ++u, ++issued) {
        const int j = j0 + u;
        const int stg = u % C::NSTG;
        const uint32_t ph = static_cast<uint32_t>(u / C::NSTG) & 1u;
        if (!W.wait(BAR(C::BAR_STE + stg), ph ^ 1u, 70)) break;
        const uint32_t dst = sbase + C::SMEM_KV + 2 * stg * C::SLOT;
        if (leader) mbar_expect_tx(BAR(C::BAR_KVF + 2 * stg), 2 * C::SLOT);
        tma_load_5d_pair(dst, &tm_k, LBAR(C::BAR_KVF + 2 * stg), 0,
                         BC * j + C::KROWS * static_cast<int>(rank), 0, hk, b);
        if ((p.debug_flags & 1) && u == 0) continue;  // test hook: drop the first V tile
        if (leader) mbar_expect_tx(BAR(C::BAR_KVF + 2 * stg + 1), 2 * C::SLOT);
        tma_load_5d_pair(dst + C::SLOT, &tm_v, LBAR(C::BAR_KVF + 2 * stg + 1), 0, BC * j,
                         C::VCH * static_cast<int>(rank), hk, b);
      }
      // rank 0's full barriers count both CTAs' bytes: draining them covers
      // the loads of rank 1 too (which leaves only after the final cluster
      // barrier, after this drain)
      if (leader) {
        W.drain(BAR(C::BAR_Q), 0, 71);
        for (int g = 0; g < C::NSTG && g < issued; ++g) {
          const int last = g + ((issued - 1 - g) / C::NSTG) * C::NSTG;
          const uint32_t ph = static_cast<uint32_t>(last / C::NSTG) & 1u;
          W.drain(BAR(C::BAR_KVF + 2 * g), ph, 72);
          W.drain(BAR(C::BAR_KVF + 2 * g + 1), ph, 73);
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------- pair products (rank 0, one thread)
    if (leader && lane == 0) {
      constexpr uint32_t idesc_s = idesc_make(256, BC, 1u, false, false);
      constexpr uint32_t idesc_o = idesc_make(256, D, 1u, false, true);
      auto kslot = [&](int u) { return 2 * (u % C::NSTG); };
      auto vslot = [&](int u) { return 2 * (u % C::NSTG) + 1; };
      auto kph = [&](int u) { return static_cast<uint32_t>(u / C::NSTG) & 1u; };
      auto vph = kph;
      // the same barrier of both CTAs, reached by one commit
      auto commit_both = [&](int i) {
#if ETA_PAIR_COMMIT_MASK
        mma_commit_pair_both(BAR(i), static_cast<uint16_t>(0x3));
#else
        mma_commit_pair(obar0 + 8u * static_cast<uint32_t>(i));
        mma_commit_pair(pbar0 + 8u * static_cast<uint32_t>(i));
#endif
      };
      const SDesc qa = sdesc_base(sbase + C::SMEM_Q, 16, 1024);
      auto issue_s = [&](int buf, int slot) {
        const SDesc kd = sdesc_base(sbase + C::SMEM_KV + slot * C::SLOT, 16, 1024);
        const uint32_t d = tmem + C::S_COL + BC * buf;
#pragma unroll
        for (int ks = 0; ks < C::QK_STEPS; ++ks) {
          const uint32_t qoff = (ks >> 2) * C::QCHUNK + (ks & 3) * 32;
          const uint32_t koff = (ks >> 2) * C::KCHUNK + (ks & 3) * 32;
          mma_ss_pair(d, sdesc_at(qa, qoff), sdesc_at(kd, koff), idesc_s, ks > 0);
        }
      };
      auto issue_pv = [&](int buf, int slot, bool acc) {
        // this CTA's V half: 64 key rows (K) x 64 D columns (its N half), MN-major
        const SDesc vd = sdesc_base(sbase + C::SMEM_KV + slot * C::SLOT, C::VHALF, 1024);
        const uint32_t a = tmem + C::S_COL + BC * buf;
#pragma unroll
        for (int ks = 0; ks < C::PV_STEPS; ++ks)
          mma_ts_pair(tmem + C::O_COL, a + 8u * ks, sdesc_at(vd, ks * 16 * 128), idesc_o,
                      ks > 0 ? 1u : (acc ? 1u : 0u));
      };
      bool ok = n > 0 && W.wait(BAR(C::BAR_Q), 0, 80) &&
                W.wait(BAR(C::BAR_KVF + kslot(0)), kph(0), 81);
      if (ok) {
        tc_fence_after();
        issue_s(0, kslot(0));
        commit_both(C::BAR_S + 0);
      }
      for (int u = 0; ok && u < n; ++u) {
        if (u + 1 < n) {
          if (!W.wait(BAR(C::BAR_KVF + kslot(u + 1)), kph(u + 1), 82)) { ok = false; break; }
          tc_fence_after();
          issue_s((u + 1) & 1, kslot(u + 1));
          commit_both(C::BAR_S + ((u + 1) & 1));
        }
        if (!W.wait(BAR(C::BAR_P + (u & 1)), (u >> 1) & 1, 83)) { ok = false; break; }
        if (!W.wait(BAR(C::BAR_KVF + vslot(u)), vph(u), 84)) { ok = false; break; }
        tc_fence_after();
        issue_pv(u & 1, vslot(u), u > 0);
        commit_both(C::BAR_STE + u % C::NSTG);  // the tile's K and V halves are free
      }
      if (ok) commit_both(C::BAR_O);
      commit_both(C::BAR_DONE);
      W.drain(BAR(C::BAR_DONE), 0, 85);
    }
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();  // no product of the pair still reads or writes either CTA
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

}  // namespace eta
