// Column-parallel dK / dV kernel with three Q stages (head dimension 128).
//
// Same method as bwd_kv_kernel (bwd_split.cuh: per 128-row key tile of one
// key/value head, a loop over the group's query heads x 128-row query tiles
// computing S^T = K Q_i^T, dP^T = V dO_i^T, P^T, dS^T = P^T (dP^T - Delta),
// dV += P^T dO_i, dK += dS^T Q_i; the atomic-free seven-product form of the
// FlashAttention (Metal Port) README, Documentation section), with the shared
// memory spent differently:
//
//  * Q_i has three stages (dO_i two): Q_i is read first by S^T(i) and last by
//    dK(i), so with two stages Q_{i+1} could only be loaded once dK(i-1) was
//    done, and S^T(i+1) waited for it (clock64 timelines of the 4096-token
//    causal backward: ~900 cycles per query tile);
//  * P^T lives in tensor memory, not shared memory: each elementwise
//    warpgroup writes its P^T columns (bf16 pairs) into the upper half of its
//    dP^T columns once it has read them, and dV += P^T dO_i reads A from
//    there; dS^T goes to the lower half as before (dK reads it);
//  * the epilogue stages its TMA stores of dK and dV in the Q stage of the
//    item's last query tile (free once dK of that tile is done); the producer
//    reloads that stage only after the epilogue's stores have read it (one
//    barrier per Q stage, so its phases cannot alias).
//
// Row statistics travel with the tile that needs them: lse2 with Q_i (for
// P^T), Delta with dO_i (for dS^T).
//
// With DS, each elementwise thread also writes its row of every tile's dS^T
// (64 bf16 values per warpgroup) to the stored-dS scratch, in the layout the
// dQ kernel of bwd_dqs.cuh copies straight into shared memory.
#pragma once

#include "bwd_dqs.cuh"

namespace eta {

// Packed TMEM column of the first element of MMA K-step ks (16 elements) of
// the upper-half layout: columns of warpgroup g (CW of them) packed two bf16
// per column starting at CW g + CW / 2.
template <int CW>
__device__ __forceinline__ constexpr uint32_t packed_col_hi(int ks) {
  return static_cast<uint32_t>((16 * ks / CW) * CW + CW / 2 + ((16 * ks) % CW) / 2);
}

template <int D, int NQ, int NO, int NWG_>
struct BwdKV3Cfg {
  static constexpr int BC = 128, BR = 128;
  static constexpr int NWG = NWG_, CW = 128 / NWG;
  static constexpr int ROWB = D * 2;
  static constexpr int NCHUNK = ROWB / 128;
  static constexpr int CHUNK = 128 * 128;
  static constexpr int TILE = 128 * ROWB;
  static constexpr int KSTEPS = ROWB / 32;
  // TMEM: S^T | dP^T (dS^T bf16 in the lower half, P^T in the upper half of
  // each warpgroup's columns) | dV | dK
  static constexpr int T_ST = 0, T_DPT = 128, T_DV = 256, T_DK = 256 + D, TMEM_COLS = 512;
  static constexpr int S_K = 0, S_V = TILE, S_Q = 2 * TILE;   // [NQ] Q tiles
  static constexpr int S_DO = S_Q + NQ * TILE;                 // [NO] dO tiles
  static constexpr int S_QST = S_DO + NO * TILE;               // [NQ] lse2[128]
  static constexpr int S_OST = S_QST + NQ * 512;               // [NO] delta[128]
  static constexpr int S_BAR = S_OST + NO * 512;
  // kv (K, V loaded), q_full[NQ] (Q_i, lse2), q_empty[NQ] (dK done),
  // do_full[NO] (dO_i, Delta), do_empty[NO] (dK done: Delta is read until
  // dS^T is complete), epi[NQ] (the
  // epilogue's stores staged in the Q stage have read it), s, s_consumed,
  // dp, p, ds, kv_done (dK, dV complete), done, kv_empty (K, V no longer read)
  static constexpr int B_KV = 0, B_QF = 1, B_QE = 1 + NQ, B_OF = 1 + 2 * NQ,
                       B_OE = 1 + 2 * NQ + NO, B_EPI = 1 + 2 * NQ + 2 * NO,
                       B_S = 1 + 3 * NQ + 2 * NO, B_SC = B_S + 1, B_DP = B_S + 2, B_P = B_S + 3,
                       B_DS = B_S + 4, B_KVD = B_S + 5, B_DONE = B_S + 6, B_KVE = B_S + 7,
                       NBAR = B_S + 8;
  static constexpr int S_MISC = S_BAR + 8 * NBAR;
  static constexpr int S_META = S_MISC + 16;  // [NQ] entry index of each Q stage
  static constexpr int S_SLOT = S_META + 16;  // [NQ] its stored-dS tile slot (DS)
  static constexpr int LAYOUT = S_SLOT + 16;
  static constexpr int SMEM_BYTES = LAYOUT + 1024 <= 232448 ? LAYOUT + 1024 : 232448;
  static constexpr int PRODUCER = 4 * NWG, MMA = 4 * NWG + 1;
  static constexpr int THREADS = 128 * NWG + 64;
  static_assert(LAYOUT <= 232448, "shared memory budget");
  static_assert(NQ <= 4, "stage metadata slots");
  static_assert(NWG == 2 && D == 128, "dV / dK epilogue: one warpgroup each, 64-column boxes");
  static_assert(CW == 64, "P^T and dS^T halves of 32 packed columns");
};

template <int D, int NQ, int NO, int NWG, bool DS>
__global__ void __launch_bounds__(128 * NWG + 64, 1)
    bwd_kv3_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_dk,
                   const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using C = BwdKV3Cfg<D, NQ, NO, NWG>;
  constexpr int CW = C::CW;
  static_assert(!DS || (D == 128 && CW == 64), "stored dS^T rows of 64 queries per warpgroup");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  if (smem - smem_raw + C::LAYOUT > C::SMEM_BYTES) {
    // the 1024-byte aligned layout does not fit this block's shared memory
    if (threadIdx.x == 0 && atomicCAS(p.status, 0, kErrDeviceTimeout) == 0) p.status[1] = 299;
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::S_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::S_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::S_MISC + 4);

  // let the dQ kernel that follows start on the SMs this kernel's CTAs leave
  // as they finish (with DS it waits for this grid's completion before it
  // reads the stored tiles)
  grid_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Persistent CTAs over work items (key/value head, batch, key tile), key
  // tile slowest, dealt out in snake order (as bwd_kv_kernel).
  const int nkt = (p.N + C::BC - 1) / C::BC;
  const int items = p.Hkv * p.B * nkt;
  const bool sparse = p.bmask != nullptr;
  auto item_of = [&](int r) -> KVItem {
    const int w = snake_item(r, blockIdx.x, gridDim.x, items);
    KVItem I;
    I.valid = w >= 0;
    if (!I.valid) return I;
    I.kt = w / (p.Hkv * p.B);
    I.b = (w / p.Hkv) % p.B;
    I.hk = w % p.Hkv;
    I.k0 = I.kt * C::BC;
    const int q_lo = p.wr < 0 ? 0 : max(0, I.k0 - p.wr);
    const int q_hi = p.wl < 0 ? p.N : min(p.N, min(p.N, I.k0 + C::BC) + p.wl);
    I.i_first = q_lo / C::BR;
    I.per_head = (q_hi + C::BR - 1) / C::BR - I.i_first;
    I.E = I.per_head * p.group;
    return I;
  };
  auto head_of = [&](const KVItem& I, int e) { return I.hk * p.group + e / I.per_head; };
  auto qtile_of = [&](const KVItem& I, int e) { return I.i_first + e % I.per_head; };
  auto marked = [&](const KVItem& I, int e) -> bool {
    return p.bmask[((static_cast<long long>(I.b) * p.Hq + head_of(I, e)) * p.nt + qtile_of(I, e)) *
                       p.nt +
                   I.kt] != 0;
  };
  auto count = [&](const KVItem& I) -> int {
    if (!sparse) return I.E;
    int c = 0;
    for (int base = 0; base < I.E; base += 32)
      c += __popc(__ballot_sync(0xffffffffu, base + lane < I.E && marked(I, base + lane)));
    return c;
  };
  volatile int* meta = reinterpret_cast<volatile int*>(smem + C::S_META);
  volatile int* slot_of = reinterpret_cast<volatile int*>(smem + C::S_SLOT);
#ifdef ETA_TRACE
  const int tcta = blockIdx.x == 0 ? 0 : (blockIdx.x == 1 ? 1 : -1);
#else
  const int tcta = -1;
#endif
  (void)tcta;

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_KV), 1);
    mbar_init(BAR(C::B_KVE), 1);
    for (int s = 0; s < NQ; ++s) {
      mbar_init(BAR(C::B_QF + s), 1);
      mbar_init(BAR(C::B_QE + s), 1);
      mbar_init(BAR(C::B_EPI + s), 4 * NWG);
    }
    for (int s = 0; s < NO; ++s) {
      mbar_init(BAR(C::B_OF + s), 1);
      mbar_init(BAR(C::B_OE + s), 1);
    }
    mbar_init(BAR(C::B_S), 1);
    mbar_init(BAR(C::B_SC), 4 * NWG);
    mbar_init(BAR(C::B_DP), 1);
    mbar_init(BAR(C::B_P), 4 * NWG);
    mbar_init(BAR(C::B_DS), 4 * NWG);
    mbar_init(BAR(C::B_KVD), 1);
    mbar_init(BAR(C::B_DONE), 1);
    *abort_flag = 0u;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == C::MMA) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, p.status, p.wait_limit_ns};
  // Barrier phases run on across items: g counts computed entries (query
  // tiles) of all items so far; K/V and dK/dV barriers count items that
  // compute at least one entry; epi[s] counts the epilogues staged in stage s.

  if (warp < 4 * NWG) {
    // ---------------------------------------- P^T, dS^T rows (thread j = key row j)
    const int par = warp >> 2;  // query columns [CW par, CW par + CW) of each tile
    const int j = threadIdx.x & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t st_addr = tmem + lane_base + C::T_ST + CW * par;
    const uint32_t dpt_addr = tmem + lane_base + C::T_DPT + CW * par;
    bool ok = true;
    int g = 0, nkvd = 0;
    for (int r = 0; ok; ++r) {
      const KVItem I = item_of(r);
      if (!I.valid) break;
      const int n = count(I);
      const int jg = I.k0 + j;
      for (int it = 0; it < n; ++it, ++g) {
        const int qs = g % NQ, os = g % NO;
        if (!W.wait_warp(BAR(C::B_S), g & 1, 230)) { ok = false; break; }
        // (complete already: S^T was computed from this stage) orders the reads
        // of the stage's entry index and lse2 after the producer's writes
        if (!W.wait_warp(BAR(C::B_QF + qs), (g / NQ) & 1, 234)) { ok = false; break; }
        if (j == 0) ETA_TRACE_AT(tcta, par & 1, g, 0);
        tc_fence_after();
        float pr[CW];
        tmem_load_row<CW>(st_addr, pr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_SC));  // S^T may be overwritten
        const float* lse2 = reinterpret_cast<const float*>(smem + C::S_QST + qs * 512) + CW * par;
        // (read now: the producer rewrites the slot once dK of this entry is done)
        const int ecur = meta[qs];
        const int ig0 = qtile_of(I, ecur) * C::BR + CW * par;
        // window: query ig0 + i sees key jg iff jg - wr <= ig0 + i <= jg + wl
        const int ilo = p.wr < 0 ? -(1 << 30) : jg - p.wr - ig0;
        const int ihi = p.wl < 0 ? (1 << 30) : jg + p.wl - ig0;
        const float2 c2 = make_float2(p.c, p.c);
        if (ilo <= 0 && ihi >= CW - 1) {
#pragma unroll
          for (int i = 0; i < CW; i += 2) {
            const float2 l2 = *reinterpret_cast<const float2*>(lse2 + i);
            const float2 x = ffma2(make_float2(pr[i], pr[i + 1]), c2, make_float2(-l2.x, -l2.y));
            pr[i] = ex2(x.x);
            pr[i + 1] = ex2(x.y);
          }
        } else {
#pragma unroll
          for (int i = 0; i < CW; i += 2) {
            const float2 l2 = *reinterpret_cast<const float2*>(lse2 + i);
            const float2 x = ffma2(make_float2(pr[i], pr[i + 1]), c2, make_float2(-l2.x, -l2.y));
            pr[i] = (i < ilo || i > ihi) ? 0.f : ex2(x.x);
            pr[i + 1] = (i + 1 < ilo || i + 1 > ihi) ? 0.f : ex2(x.y);
          }
        }
        // dP^T(g) is complete (and with it, in issue order, every product that
        // read the previous tile's P^T and dS^T from these columns)
        if (!W.wait_warp(BAR(C::B_DP), g & 1, 231)) { ok = false; break; }
        if (j == 0) ETA_TRACE_AT(tcta, par & 1, g, 2);
        // (complete already: dP^T was computed from this stage) orders the
        // reads of Delta after the producer's writes
        if (!W.wait_warp(BAR(C::B_OF + os), (g / NO) & 1, 235)) { ok = false; break; }
        tc_fence_after();
        const float* dlt = reinterpret_cast<const float*>(smem + C::S_OST + os * 512) + CW * par;
        // dS^T = P^T (dP^T - Delta) of the upper half of this warpgroup's dP^T
        // columns first, so that they can take P^T (bf16 pairs): the A
        // operand of dV += P^T dO_i
        uint32_t dk[32];
        {
          uint32_t rh[32];
          tmem_ld32(dpt_addr + CW / 2, rh);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 dd = *reinterpret_cast<const float2*>(dlt + 32 + i);
            const float2 gd = fsub2(make_float2(u2f(rh[i]), u2f(rh[i + 1])), dd);
            dk[16 + i / 2] = pack_bf16x2(pr[32 + i] * gd.x, pr[32 + i + 1] * gd.y);
          }
        }
        {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(pr[2 * i], pr[2 * i + 1]);
          tmem_st32(dpt_addr + CW / 2, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_P));
        if (j == 0) ETA_TRACE_AT(tcta, par & 1, g, 1);
        // stored dS^T (see below): this key's values of the upper 32 queries
        // now, the lower 32 once they are computed (two bursts of stores).
        // The entry's tile slot comes from the load warp (read before this
        // thread's dS^T hand-off, after which the stage may be reloaded)
        int dslot = 0;
        auto ds_row = [&]() -> uint8_t* {
          return p.ds + static_cast<long long>(dslot) * kDsTileBytes + par * (kDsTileBytes / 2) +
                 j * 16;
        };
        if constexpr (DS) {
          dslot = slot_of[qs];
          uint8_t* trow = ds_row();
#pragma unroll
          for (int m = 4; m < 8; ++m)
            *reinterpret_cast<uint4*>(trow + m * 2048) =
                make_uint4(dk[4 * m], dk[4 * m + 1], dk[4 * m + 2], dk[4 * m + 3]);
        }
        // the lower half
        {
          uint32_t rl[32];
          tmem_ld32(dpt_addr, rl);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 dd = *reinterpret_cast<const float2*>(dlt + i);
            const float2 gd = fsub2(make_float2(u2f(rl[i]), u2f(rl[i + 1])), dd);
            dk[i / 2] = pack_bf16x2(pr[i] * gd.x, pr[i + 1] * gd.y);
          }
        }
        // dS^T (bf16 pairs) into the lower half: the A operand of dK += dS^T Q_i
        tmem_st32(dpt_addr, dk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_DS));
        if constexpr (DS) {
          // this key's dS^T values into the stored tile: queries 8 m .. 8 m + 7
          // of this warpgroup's 64 form query group 8 par + m (2 KB apart),
          // row j (16 bytes); a warp's 32 keys write 512 contiguous bytes
          uint8_t* trow = ds_row();
#pragma unroll
          for (int m = 0; m < 4; ++m)
            *reinterpret_cast<uint4*>(trow + m * 2048) =
                make_uint4(dk[4 * m], dk[4 * m + 1], dk[4 * m + 2], dk[4 * m + 3]);
        }
        if (j == 0) ETA_TRACE_AT(tcta, par & 1, g, 3);
      }
      if (!ok) break;
      // epilogue: warpgroup 0 stores dV, warpgroup 1 dK x scale (128 columns
      // each), through TMA stores staged in the Q stage of the item's last
      // entry; then that stage is released to the producer
      const int which = par;
      if (n > 0) {
        if (!W.wait_warp(BAR(C::B_KVD), nkvd & 1, 232)) { ok = false; break; }
        ++nkvd;
        tc_fence_after();
        const int ls = (g - 1) % NQ;  // Q stage of the item's last entry
        uint8_t* stage = smem + C::S_Q + ls * C::TILE + par * C::CHUNK + (warp & 3) * 32 * 128;
        const uint32_t src = tmem + lane_base + (which ? C::T_DK : C::T_DV);
        tmem_rows_tma_store<D>(src, stage, which ? &tm_dk : &tm_dv, 0, I.k0 + (warp & 3) * 32,
                               I.hk, I.b, which ? p.scale : 1.f);
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_EPI + ls));
      } else if (jg < p.N) {
        // no query sees these keys: their gradients are zero
        __nv_bfloat16* row =
            which == 0 ? static_cast<__nv_bfloat16*>(p.dv) + I.b * p.dvsb + I.hk * p.dvsh +
                             static_cast<long long>(jg) * p.dvsn
                       : static_cast<__nv_bfloat16*>(p.dk) + I.b * p.dksb + I.hk * p.dksh +
                             static_cast<long long>(jg) * p.dksn;
        for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(row)[c] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  } else if (warp == C::PRODUCER) {
    // ---------------------------------------- TMA producer (the whole warp scans
    // 32 entries at a time; lane 0 waits and issues the copies)
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
    }
    int g = 0, m = 0, issued_q = 0, issued_do = 0;
    // per Q stage (bit s): whether its previous entry was the last of an item
    // (whose epilogue stages its stores there), and the parity of the number
    // of such epilogues so far
    uint32_t epi_pending = 0u, epi_parity = 0u;
    bool pok = true;
    for (int r = 0; pok; ++r) {
      const KVItem I = item_of(r);
      if (!I.valid) break;
      const int nI = count(I);
      int done_in_item = 0;
      bool kv_loaded = false;
      for (int base = 0; pok && base < I.E; base += 32) {
        const int e_l = base + lane;
        const bool on = e_l < I.E && (!sparse || marked(I, e_l));
        uint32_t pend = __ballot_sync(0xffffffffu, on);
        while (pend != 0u) {
          const int e = base + __ffs(pend) - 1;
          pend &= pend - 1u;
          if (lane == 0) {
            if (!kv_loaded) {
              if (m > 0 && !W.wait(BAR(C::B_KVE), (m - 1) & 1, 245)) {
                pok = false;
              } else {
                // K, V are read by this item only (L2 evict first); Q, dO by
                // the items of every key tile of the head (evict last)
                mbar_expect_tx(BAR(C::B_KV), 2 * C::TILE);
                for (int c = 0; c < C::NCHUNK; ++c) {
                  tma_load_4d_hint(sbase + C::S_K + c * C::CHUNK, &tm_k, BAR(C::B_KV), c * 64,
                                   I.k0, I.hk, I.b, l2_policy_evict_first());
                  tma_load_4d_hint(sbase + C::S_V + c * C::CHUNK, &tm_v, BAR(C::B_KV), c * 64,
                                   I.k0, I.hk, I.b, l2_policy_evict_first());
                }
                ++m;
              }
              kv_loaded = true;
            }
            const int qs = g % NQ, os = g % NO;
            const int h = head_of(I, e);
            const int ig0 = qtile_of(I, e) * C::BR;
            const long long srow = static_cast<long long>(I.b * p.Hq + h) * p.Npad + ig0;
            // Q_i first: with three stages its slot is free long before dO_i's
            // (which waits for dK two tiles back), and S^T(i) needs it first
            if (pok) {
              bool qfree = W.wait(BAR(C::B_QE + qs), ((g / NQ) & 1) ^ 1, 240);
              if (qfree && ((epi_pending >> qs) & 1u)) {
                // the stage held an item's last entry: its epilogue's stores
                // must have read it
                qfree = W.wait(BAR(C::B_EPI + qs), (epi_parity >> qs) & 1u, 246);
                epi_pending &= ~(1u << qs);
                epi_parity ^= 1u << qs;
              }
              if (!qfree) {
                pok = false;
              } else {
                ETA_TRACE_AT(tcta, 3, g, 0);
                meta[qs] = e;
                if constexpr (DS) slot_of[qs] = static_cast<int>(ds_slot(p, I.b, h, qtile_of(I, e), I.kt));
                const uint32_t full = BAR(C::B_QF + qs);
                mbar_expect_tx(full, C::TILE + 512);
                for (int c = 0; c < C::NCHUNK; ++c)
                  if (!((p.debug_flags & 2) && g == 1))
                    tma_load_4d_hint(sbase + C::S_Q + qs * C::TILE + c * C::CHUNK, &tm_q, full,
                                     c * 64, ig0, h, I.b, l2_policy_evict_last());
                bulk_load(sbase + C::S_QST + qs * 512, p.lse2 + srow, 512, full);
                issued_q = g + 1;
                if (++done_in_item == nI) epi_pending |= 1u << qs;
              }
            }
            if (pok) {
              if (!W.wait(BAR(C::B_OE + os), ((g / NO) & 1) ^ 1, 243)) {
                pok = false;
              } else {
                const uint32_t ofull = BAR(C::B_OF + os);
                mbar_expect_tx(ofull, C::TILE + 512);
                for (int c = 0; c < C::NCHUNK; ++c)
                  tma_load_4d_hint(sbase + C::S_DO + os * C::TILE + c * C::CHUNK, &tm_do, ofull,
                                   c * 64, ig0, h, I.b, l2_policy_evict_last());
                bulk_load(sbase + C::S_OST + os * 512, p.delta + srow, 512, ofull);
                issued_do = g + 1;
              }
            }
          }
          pok = __shfl_sync(0xffffffffu, pok, 0);
          if (!pok) break;
          ++g;
        }
      }
    }
    if (lane == 0) {
      if (m > 0) W.drain(BAR(C::B_KV), static_cast<uint32_t>(m - 1) & 1u, 241);
      for (int s = 0; s < NQ && s < issued_q; ++s) {
        const int last = s + ((issued_q - 1 - s) / NQ) * NQ;
        W.drain(BAR(C::B_QF + s), static_cast<uint32_t>(last / NQ) & 1u, 242);
      }
      for (int s = 0; s < NO && s < issued_do; ++s) {
        const int last = s + ((issued_do - 1 - s) / NO) * NO;
        W.drain(BAR(C::B_OF + s), static_cast<uint32_t>(last / NO) & 1u, 244);
      }
    }
    __syncwarp();
  } else if (warp == C::MMA) {
    // ---------------------------------------- MMA issuer (whole warp, one elected lane issues)
    constexpr uint32_t id_s = idesc_make(128, 128, 1u, false, false);  // S^T, dP^T
    constexpr uint32_t id_kv = idesc_make(128, D, 1u, false, true);    // dV, dK
    const SDesc dK = sdesc_base(sbase + C::S_K, 16, 1024);
    const SDesc dV = sdesc_base(sbase + C::S_V, 16, 1024);
    auto issue_s = [&](int g) -> bool {
      const int qs = g % NQ;
      if (!W.wait_warp(BAR(C::B_QF + qs), (g / NQ) & 1, 250)) return false;
      tc_fence_after();
      const SDesc dq = sdesc_base(sbase + C::S_Q + qs * C::TILE, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
        mma_ss_w(tmem + C::T_ST, sdesc_at(dK, off), sdesc_at(dq, off), id_s, ks > 0);
      }
      mma_commit_w(BAR(C::B_S));
      return true;
    };
    auto issue_dp = [&](int g) -> bool {
      const int os = g % NO;
      if (!W.wait_warp(BAR(C::B_OF + os), (g / NO) & 1, 256)) return false;
      tc_fence_after();
      const SDesc ddo = sdesc_base(sbase + C::S_DO + os * C::TILE, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
        mma_ss_w(tmem + C::T_DPT, sdesc_at(dV, off), sdesc_at(ddo, off), id_s, ks > 0);
      }
      mma_commit_w(BAR(C::B_DP));
      return true;
    };
    bool ok = true;
    int g = 0, nkv = 0;
    for (int r = 0; ok; ++r) {
      const KVItem I = item_of(r);
      if (!I.valid) break;
      const int n = count(I);
      if (n == 0) continue;
      if (!W.wait_warp(BAR(C::B_KV), nkv & 1, 251)) { ok = false; break; }
      ++nkv;
      // the item's first S^T overwrites S^T of the previous item's last entry
      if (g > 0 && !W.wait_warp(BAR(C::B_SC), (g - 1) & 1, 257)) { ok = false; break; }
      if (!issue_s(g) || !issue_dp(g)) { ok = false; break; }
      if (n == 1) mma_commit_w(BAR(C::B_KVE));  // K and V are not read again
      for (int it = 0; it < n; ++it, ++g) {
        const int qs = g % NQ, os = g % NO;
        const uint32_t acc0 = it > 0 ? 1u : 0u;
        ETA_TRACE_AT(tcta, 2, g, 0);
        // S^T of the next tile once the elementwise warps have loaded this one
        if (it + 1 < n) {
          if (!W.wait_warp(BAR(C::B_SC), g & 1, 255)) { ok = false; break; }
          ETA_TRACE_AT(tcta, 3, g, 1);
          if (!issue_s(g + 1)) { ok = false; break; }
        }
        ETA_TRACE_AT(tcta, 2, g, 1);
        // dV += P^T dO_i: A = P^T (TMEM, upper halves of the dP^T columns),
        // B = dO_i (MN-major)
        if (!W.wait_warp(BAR(C::B_P), g & 1, 252)) { ok = false; break; }
        ETA_TRACE_AT(tcta, 2, g, 2);
        tc_fence_after();
        const SDesc ddo = sdesc_base(sbase + C::S_DO + os * C::TILE, C::CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_w(tmem + C::T_DV, tmem + C::T_DPT + packed_col_hi<CW>(ks),
                   sdesc_at(ddo, ks * 2048), id_kv, ks > 0 ? 1u : acc0);
        ETA_TRACE_AT(tcta, 3, g, 2);
        // dK += dS^T Q_i with dS^T from TMEM (lower halves)
        if (!W.wait_warp(BAR(C::B_DS), g & 1, 253)) { ok = false; break; }
        ETA_TRACE_AT(tcta, 2, g, 3);
        tc_fence_after();
        const SDesc dq = sdesc_base(sbase + C::S_Q + qs * C::TILE, C::CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_w(tmem + C::T_DK, tmem + C::T_DPT + packed_col<CW>(ks), sdesc_at(dq, ks * 2048),
                   id_kv, ks > 0 ? 1u : acc0);
        // dO_i is last read by dV(i), but its stage also holds Delta_i, which
        // the elementwise warps read for the second half of dS^T after they
        // have released P^T (and with it dV(i)): the stage is free only once
        // their dS^T is in, i.e. after dK(i)
        mma_commit_w(BAR(C::B_OE + os));
        mma_commit_w(BAR(C::B_QE + qs));  // Q_i (and lse2) are not read again
        if (it + 1 < n) {
          if (!issue_dp(g + 1)) { ok = false; break; }
          if (it + 2 == n) mma_commit_w(BAR(C::B_KVE));  // K and V are not read again
        }
        ETA_TRACE_AT(tcta, 3, g, 3);
      }
      if (!ok) break;
      mma_commit_w(BAR(C::B_KVD));  // dK, dV of this item complete
    }
    mma_commit_w(BAR(C::B_DONE));
    W.drain(BAR(C::B_DONE), 0, 254);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace eta
