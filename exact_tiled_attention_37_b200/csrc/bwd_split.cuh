// Atomic-free backward for head dimensions 64 and 128: the alternative the
// FlashAttention (Metal Port) README describes (Documentation section: seven
// products instead of five, full parallelism over both the rows and the
// columns of the attention matrix, no atomics):
//
//  * bwd_q_kernel (row-parallel): per 128-row query tile, loop over 128-row
//    key tiles: S = Q K_j^T, dP = dO V_j^T, P = exp2(S c - lse2),
//    dS = P (dP - Delta), dQ += dS K_j; dQ is written once, in bf16.
//  * bwd_kv_kernel (column-parallel): per 128-row key tile, loop over the
//    query heads of the group x 128-row query tiles: S^T = K Q_i^T,
//    dP^T = V dO_i^T, P^T, dS^T, dV += P^T dO_i, dK += dS^T Q_i.  Persistent:
//    one CTA per SM walks its share of the key tiles (a static snake order
//    over tiles sorted by work), with barrier phases carried from one key
//    tile to the next, and writes dK, dV through TMA stores.
//
// Both read lse2 = lse log2(e) and Delta = rowsum(dO O) from the
// preprocess kernel.  All MMAs are M = 128, N = 128 (or D) shapes, issued
// by one whole warp (one elected lane issues each instruction).  NWG
// elementwise warpgroups split the 128 columns of every tile: warpgroup g
// owns columns [CW g, CW g + CW), CW = 128 / NWG, and thread t of it owns
// row t (its TMEM lane).  A bf16 tile written back into TMEM keeps column c
// of warpgroup g at packed column CW g + (c - CW g) / 2.
#pragma once

#include "bwd.cuh"
#include "fwd.cuh"

namespace eta {

// Packed TMEM column of the first element of MMA K-step ks (16 elements)
// when the 128 columns were split into groups of CW and each group packed
// two bf16 per column at its own start.
template <int CW>
__device__ __forceinline__ constexpr uint32_t packed_col(int ks) {
  return static_cast<uint32_t>((16 * ks / CW) * CW + ((16 * ks) % CW) / 2);
}

// NC fp32 TMEM columns of this thread's lane, times mul, as bf16 to row[0..NC).
template <int NC>
__device__ __forceinline__ void tmem_row_to_bf16(uint32_t taddr, __nv_bfloat16* row, float mul,
                                                 bool valid) {
  static_assert(NC % 16 == 0, "16-column chunks");
#pragma unroll 1
  for (int c = 0; c < NC / 16; ++c) {
    uint32_t r[16];
    tmem_ld16(taddr + 16 * c, r);
    tmem_wait_ld();
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(row + 16 * c);
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        uint4 w;
        w.x = pack_bf16x2(u2f(r[8 * v + 0]) * mul, u2f(r[8 * v + 1]) * mul);
        w.y = pack_bf16x2(u2f(r[8 * v + 2]) * mul, u2f(r[8 * v + 3]) * mul);
        w.z = pack_bf16x2(u2f(r[8 * v + 4]) * mul, u2f(r[8 * v + 5]) * mul);
        w.w = pack_bf16x2(u2f(r[8 * v + 6]) * mul, u2f(r[8 * v + 7]) * mul);
        dst[v] = w;
      }
    }
  }
}

// Stores CW/2 packed columns (CW = 32 or 64).
template <int CW>
__device__ __forceinline__ void tmem_store_packed(uint32_t taddr, const uint32_t (&pk)[CW / 2]) {
  if constexpr (CW == 64) {
    tmem_st32(taddr, pk);
  } else {
    tmem_st16(taddr, pk);
  }
}

// ============================================================ dQ kernel
// K_j is read by S(j) and, last, by dQ(j); V_j only by dP(j), which comes
// early.  So K and V have rings of their own: V_{j+1} reuses the slot of
// V_{j-1} (free since dP(j-1)) instead of waiting, in one shared ring, for a
// K tile that dQ still reads (clock64 timelines of the 4096-token causal
// backward: the MMA warp waited ~1.5k cycles per key tile for V_{j+1} there).
template <int D, int NK_, int NV_, int NWG_>
struct BwdQCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int NWG = NWG_, CW = 128 / NWG;
  static constexpr int ROWB = D * 2;
  static constexpr int NCHUNK = ROWB / 128;
  static constexpr int CHUNK = 128 * 128;
  static constexpr int TILE = 128 * ROWB;
  static constexpr int KSTEPS = ROWB / 32;      // S, dP over D
  static constexpr int NK = NK_, NV = NV_;      // K ring and V ring slots
  // TMEM: S[2] (128 each; dS bf16 written back) | dP | dQ
  static constexpr int T_S = 0, T_DP = 256, T_DQ = 384, TMEM_COLS = 512;
  static constexpr int SMEM_Q = 0, SMEM_DO = TILE, SMEM_K = 2 * TILE;
  static constexpr int SMEM_V = SMEM_K + NK * TILE;
  static constexpr int SMEM_BAR = SMEM_V + NV * TILE;
  // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2],
  // dp_full, ds_full[2], dq_done, done, dp_consumed.  ds_full alternates by
  // key tile: a warp may arrive for tile u + 1 (it needs only dP(u) loaded by
  // every warp, not dS(u) written) before the last warp arrives for tile u.
  static constexpr int B_Q = 0, B_KF = 1, B_KE = 1 + NK, B_VF = 1 + 2 * NK,
                       B_VE = 1 + 2 * NK + NV, B_S = 1 + 2 * NK + 2 * NV,
                       B_DP = B_S + 2, B_DS = B_S + 3, B_DQ = B_S + 5, B_DONE = B_S + 6,
                       B_DPC = B_S + 7, NBAR = B_S + 8;
  static constexpr int SMEM_MISC = SMEM_BAR + 8 * NBAR;
  static constexpr int SMEM_BITS = SMEM_MISC + 16;  // block-sparse: computed key tiles
  static constexpr int SMEM_BYTES = SMEM_BITS + 4 * kMaskWords + 1024;
  static constexpr int PRODUCER = 4 * NWG, MMA = 4 * NWG + 1;  // warp indices
  static constexpr int THREADS = 128 * NWG + 64;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(D % (16 * NWG) == 0, "dQ columns per warpgroup");
};

template <int D, int NK, int NV, int NWG>
__global__ void __launch_bounds__(128 * NWG + 64, 1)
    bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_dq,
                 const BwdParams p) {
  using C = BwdQCfg<D, NK, NV, NWG>;
  constexpr int CW = C::CW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::SMEM_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid order as the forward's (FwdParams::head_major)
  const int qb = p.head_major ? gridDim.x - 1 - blockIdx.x : gridDim.z - 1 - blockIdx.z;
  const int h = p.head_major ? blockIdx.y : blockIdx.x;
  const int b = p.head_major ? blockIdx.z : blockIdx.y;
  const int hk = h / p.group;
  const int q0 = qb * C::BM;
  const int2 ktr = key_tiles(q0, p.N, p.wl, p.wr, C::BN);
  const int jlo = ktr.x, jhi = ktr.y;  // key tiles in the window range
  // Block-sparse: bit j marks key tile j as computed for this query tile.
  const bool sparse = p.bmask != nullptr;
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + C::SMEM_BITS);
  if (sparse) {
    for (int wi = warp; wi < kMaskWords; wi += C::THREADS / 32) {
      const int j = 32 * wi + lane;
      const bool on = j >= jlo && j < jhi && qb < p.nt &&
                      p.bmask[((static_cast<long long>(b) * p.Hq + h) * p.nt + qb) * p.nt + j] != 0;
      const uint32_t w = __ballot_sync(0xffffffffu, on);
      if (lane == 0) bits[wi] = w;
    }
  }
  // first computed key tile >= j (jhi if none)
  auto next_key = [&](int j) -> int {
    j = max(j, jlo);
    return sparse ? next_bit(bits, j, jhi) : min(j, jhi);
  };
#ifdef ETA_TRACE
  const int tcta = (blockIdx.x == 0 && blockIdx.y == 0) ? (qb == 31 ? 0 : (qb == 15 ? 1 : -1)) : -1;
#else
  const int tcta = -1;
#endif
  (void)tcta;

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_Q), 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(BAR(C::B_KF + s), 1);
      mbar_init(BAR(C::B_KE + s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(BAR(C::B_VF + s), 1);
      mbar_init(BAR(C::B_VE + s), 1);
    }
    mbar_init(BAR(C::B_S + 0), 1);
    mbar_init(BAR(C::B_S + 1), 1);
    mbar_init(BAR(C::B_DP), 1);
    mbar_init(BAR(C::B_DS + 0), 4 * NWG);
    mbar_init(BAR(C::B_DS + 1), 4 * NWG);
    mbar_init(BAR(C::B_DPC), 4 * NWG);
    mbar_init(BAR(C::B_DQ), 1);
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
  // computed key tiles, in increasing order: iteration u handles the u-th
  const int n = sparse ? bits_below(bits, jhi) : jhi - jlo;

  if (warp < 4 * NWG) {
    // ---------------------------------------- dS rows (thread r = query row r), then dQ
    const int par = warp >> 2;             // key columns [CW par, CW par + CW) of each tile
    const int r = threadIdx.x & 127;
    const int qrow = q0 + r;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const long long srow = static_cast<long long>(b * p.Hq + h) * p.Npad + qrow;
    const float lse2 = p.lse2[srow];       // +inf for padded rows: their P is exactly 0
    const float dlt = p.delta[srow];
    bool ok = true;
    for (int u = 0, j = next_key(jlo); u < n; ++u, j = next_key(j + 1)) {
      const int buf = u & 1;
      const uint32_t s_addr = tmem + lane_base + C::T_S + 128 * buf + CW * par;
      if (!W.wait_warp(BAR(C::B_S + buf), (u >> 1) & 1, 100)) { ok = false; break; }
      if (r == 0) ETA_FTRACE_AT(tcta, par & 1, u, 0);
      tc_fence_after();
      float s[CW];
      tmem_load_row<CW>(s_addr, s);
      const int2 cw = col_window(C::BN * j + CW * par, qrow, p.N, p.wl, p.wr);
      const float2 c2 = make_float2(p.c, p.c), nl2 = make_float2(-lse2, -lse2);
      if (cw.x <= 0 && cw.y >= CW) {
#pragma unroll
        for (int i = 0; i < CW; i += 2) {
          const float2 x = ffma2(make_float2(s[i], s[i + 1]), c2, nl2);
          s[i] = ex2(x.x);
          s[i + 1] = ex2(x.y);
        }
      } else {
#pragma unroll
        for (int i = 0; i < CW; i += 2) {
          const float2 x = ffma2(make_float2(s[i], s[i + 1]), c2, nl2);
          s[i] = (i < cw.x || i >= cw.y) ? 0.f : ex2(x.x);
          s[i + 1] = (i + 1 < cw.x || i + 1 >= cw.y) ? 0.f : ex2(x.y);
        }
      }
      if (r == 0) ETA_FTRACE_AT(tcta, par & 1, u, 1);
      if (!W.wait_warp(BAR(C::B_DP), u & 1, 101)) { ok = false; break; }
      // dP(u) is complete, so V_u's slot is free: released from here rather
      // than by a commit of its own
      if (threadIdx.x == 0) mbar_arrive(BAR(C::B_VE + u % NV));
      if (r == 0) ETA_FTRACE_AT(tcta, par & 1, u, 2);
      tc_fence_after();
      float dp[CW];
      tmem_load_row<CW>(tmem + lane_base + C::T_DP + CW * par, dp);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_DPC));  // dP may be overwritten
      uint32_t pk[CW / 2];
      const float2 d2 = make_float2(dlt, dlt);
#pragma unroll
      for (int i = 0; i < CW; i += 2) {
        const float2 g = fsub2(make_float2(dp[i], dp[i + 1]), d2);
        pk[i / 2] = pack_bf16x2(s[i] * g.x, s[i + 1] * g.y);
      }
      // dS (bf16 pairs) into the first CW/2 of this group's S columns
      tmem_store_packed<CW>(s_addr, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_DS + (u & 1)));
      if (r == 0) ETA_FTRACE_AT(tcta, par & 1, u, 3);
    }
    // dQ * scale in bf16: warpgroup par stores columns [D/NWG par, D/NWG (par + 1))
    constexpr int DC = D / NWG;
    __nv_bfloat16* row = static_cast<__nv_bfloat16*>(p.dq) + b * p.dqsb + h * p.dqsh +
                         static_cast<long long>(qrow) * p.dqsn + DC * par;
    if (ok && n > 0 && W.wait_warp(BAR(C::B_DQ), 0, 102)) {
      tc_fence_after();
      if constexpr (DC == 64) {
        // through TMA stores, staged in this warp's rows of Q's chunk `par`
        // (every MMA reading Q is complete)
        uint8_t* stage = smem + C::SMEM_Q + par * C::CHUNK + (warp & 3) * 32 * 128;
        tmem_rows_tma_store<DC>(tmem + lane_base + C::T_DQ + DC * par, stage, &tm_dq, DC * par,
                                q0 + (warp & 3) * 32, h, b, p.scale);
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
      } else {
        tmem_row_to_bf16<DC>(tmem + lane_base + C::T_DQ + DC * par, row, p.scale, qrow < p.N);
      }
    } else if (n == 0 && qrow < p.N) {
      // no key tile is computed for this query tile: dQ = 0
      for (int c = 0; c < DC / 8; ++c) reinterpret_cast<uint4*>(row)[c] = make_uint4(0u, 0u, 0u, 0u);
    }
  } else if (warp == C::PRODUCER) {
    // ---------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_expect_tx(BAR(C::B_Q), 2 * C::TILE);
      // Q, dO are read by this CTA only (L2 evict first); K, V by every query
      // tile of the head (evict last): DRAM reads of the 2x16x4096 causal
      // backward's dQ kernel 217 -> 187 MB, time unchanged
      const uint64_t pol_once = l2_policy_evict_first(), pol_kv = l2_policy_evict_last();
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d_hint(sbase + C::SMEM_Q + c * C::CHUNK, &tm_q, BAR(C::B_Q), c * 64, q0, h, b,
                         pol_once);
        tma_load_4d_hint(sbase + C::SMEM_DO + c * C::CHUNK, &tm_do, BAR(C::B_Q), c * 64, q0, h, b,
                         pol_once);
      }
      int issued_k = 0, issued_v = 0;  // tiles whose K (V) load was issued
      for (int u = 0, j = next_key(jlo); u < n && !W.aborted(); ++u, j = next_key(j + 1)) {
        const int ks = u % NK, vs = u % NV;
        if (!W.wait(BAR(C::B_KE + ks), (static_cast<uint32_t>(u / NK) & 1u) ^ 1u, 110)) break;
        mbar_expect_tx(BAR(C::B_KF + ks), C::TILE);
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d_hint(sbase + C::SMEM_K + ks * C::TILE + c * C::CHUNK, &tm_k,
                           BAR(C::B_KF + ks), c * 64, C::BN * j, hk, b, pol_kv);
        issued_k = u + 1;
        if (!W.wait(BAR(C::B_VE + vs), (static_cast<uint32_t>(u / NV) & 1u) ^ 1u, 113)) break;
        mbar_expect_tx(BAR(C::B_VF + vs), C::TILE);
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d_hint(sbase + C::SMEM_V + vs * C::TILE + c * C::CHUNK, &tm_v,
                           BAR(C::B_VF + vs), c * 64, C::BN * j, hk, b, pol_kv);
        issued_v = u + 1;
      }
      W.drain(BAR(C::B_Q), 0, 111);
      for (int s = 0; s < NK && s < issued_k; ++s) {
        const int last = s + ((issued_k - 1 - s) / NK) * NK;
        W.drain(BAR(C::B_KF + s), static_cast<uint32_t>(last / NK) & 1u, 112);
      }
      for (int s = 0; s < NV && s < issued_v; ++s) {
        const int last = s + ((issued_v - 1 - s) / NV) * NV;
        W.drain(BAR(C::B_VF + s), static_cast<uint32_t>(last / NV) & 1u, 114);
      }
    }
    __syncwarp();
  } else if (warp == C::MMA) {
    // ---------------------------------------- MMA issuer (whole warp, one elected lane issues)
    constexpr uint32_t id_s = idesc_make(128, 128, 1u, false, false);  // S, dP
    constexpr uint32_t id_q = idesc_make(128, D, 1u, false, true);     // dQ += dS K
    const SDesc dq_ = sdesc_base(sbase + C::SMEM_Q, 16, 1024);
    const SDesc ddo = sdesc_base(sbase + C::SMEM_DO, 16, 1024);
    auto kslot = [&](int u) { return u % NK; };
    auto kph = [&](int u) { return static_cast<uint32_t>(u / NK) & 1u; };
    auto vslot = [&](int u) { return u % NV; };
    auto vph = [&](int u) { return static_cast<uint32_t>(u / NV) & 1u; };
    // S(u) = Q K^T into S[u % 2]
    auto issue_s = [&](int u) -> bool {
      if (!W.wait_warp(BAR(C::B_KF + kslot(u)), kph(u), 120)) return false;
      tc_fence_after();
      const SDesc kb = sdesc_base(sbase + C::SMEM_K + kslot(u) * C::TILE, 16, 1024);
      const uint32_t d = tmem + C::T_S + 128 * (u & 1);
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
        mma_ss_w(d, sdesc_at(dq_, off), sdesc_at(kb, off), id_s, ks > 0);
      }
      mma_commit_w(BAR(C::B_S + (u & 1)));
      return true;
    };
    // dP(u) = dO V^T
    auto issue_dp = [&](int u) -> bool {
      if (!W.wait_warp(BAR(C::B_VF + vslot(u)), vph(u), 121)) return false;
      tc_fence_after();
      const SDesc vb = sdesc_base(sbase + C::SMEM_V + vslot(u) * C::TILE, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
        mma_ss_w(tmem + C::T_DP, sdesc_at(ddo, off), sdesc_at(vb, off), id_s, ks > 0);
      }
      mma_commit_w(BAR(C::B_DP));  // also frees V_u's slot (elementwise thread 0 arrives)
      return true;
    };
    bool ok = W.wait_warp(BAR(C::B_Q), 0, 122);
    if (ok && n > 0) ok = issue_s(0) && issue_dp(0);
    if (ok && n > 1) ok = issue_s(1);
    for (int u = 0; ok && u < n; ++u) {
      // dP(u + 1) as soon as the elementwise warps have loaded dP(u)
      if (u + 1 < n) {
        if (!W.wait_warp(BAR(C::B_DPC), u & 1, 125)) { ok = false; break; }
        if (!issue_dp(u + 1)) { ok = false; break; }
      }
      ETA_FTRACE_AT(tcta, 2, u, 2);
      // dS(u) is in S[u % 2]
      if (!W.wait_warp(BAR(C::B_DS + (u & 1)), (u >> 1) & 1, 123)) { ok = false; break; }
      ETA_FTRACE_AT(tcta, 2, u, 0);
      tc_fence_after();
      // dQ += dS K_u: A = dS from TMEM, B = K_u as an MN-major operand (N = D, K = 128 keys)
      const SDesc kb = sdesc_base(sbase + C::SMEM_K + kslot(u) * C::TILE, C::CHUNK, 1024);
      const uint32_t a = tmem + C::T_S + 128 * (u & 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_ts_w(tmem + C::T_DQ, a + packed_col<CW>(ks), sdesc_at(kb, ks * 2048), id_q,
                 (u > 0 || ks > 0) ? 1u : 0u);
      mma_commit_w(BAR(C::B_KE + kslot(u)));  // K_u is not read again
      ETA_FTRACE_AT(tcta, 2, u, 1);
      // S(u + 2) into S[u % 2] after dQ(u) has read dS(u) (issue order)
      if (u + 2 < n && !issue_s(u + 2)) { ok = false; break; }
      ETA_FTRACE_AT(tcta, 2, u, 3);
    }
    if (ok) mma_commit_w(BAR(C::B_DQ));
    mma_commit_w(BAR(C::B_DONE));
    W.drain(BAR(C::B_DONE), 0, 124);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  // Launched as a programmatic dependent of the dK/dV kernel (it reads only
  // the inputs and the preprocess's statistics, complete before that kernel
  // started): waiting here, after all the work, makes this grid's completion
  // imply the dK/dV kernel's, so later work in the stream is ordered after both.
  grid_dependency_wait();
}

// Round r of a persistent CTA's static schedule: items sorted by decreasing
// work are dealt out in snake order (CTA c takes item r G + c in even
// rounds, r G + G - 1 - c in odd ones, G CTAs), which evens out the per-CTA
// sums; -1 past the last item.
__device__ __forceinline__ int snake_item(int r, int cta, int ctas, int items) {
  const int idx = r * ctas + ((r & 1) ? ctas - 1 - cta : cta);
  return idx < items ? idx : -1;
}

// One work item of the dK/dV kernel: a 128-row key tile of one key/value
// head, and the query tiles (of every query head of its group) that see it.
struct KVItem {
  bool valid;
  int hk, b, kt, k0, i_first, per_head, E;
};

// ============================================================ dK / dV kernel
// P^T goes through shared memory (the A operand of dV += P^T dO_i) so that
// S^T of the next query tile can be computed as soon as the elementwise
// warps have loaded S^T of this one; dS^T stays in TMEM (in the dP^T
// columns it was computed from).
template <int D, int NQS, int NWG_>
struct BwdKVCfg {
  static constexpr int BC = 128, BR = 128;
  static constexpr int NWG = NWG_, CW = 128 / NWG;
  static constexpr int ROWB = D * 2;
  static constexpr int NCHUNK = ROWB / 128;
  static constexpr int CHUNK = 128 * 128;
  static constexpr int TILE = 128 * ROWB;
  static constexpr int KSTEPS = ROWB / 32;
  // TMEM: S^T | dP^T (dS^T bf16 written back) | dV | dK
  static constexpr int T_ST = 0, T_DPT = 128, T_DV = 256, T_DK = 256 + D, TMEM_COLS = 512;
  static constexpr int S_K = 0, S_V = TILE, S_Q = 2 * TILE;   // [NQS] Q tiles
  static constexpr int S_DO = S_Q + NQS * TILE;                // [NQS] dO tiles
  static constexpr int S_P = S_DO + NQS * TILE;                // P^T: 128 key rows x 128 queries bf16
  static constexpr int S_STAT = S_P + 128 * 256;               // [NQS] lse2[128], delta[128]
  static constexpr int S_BAR = S_STAT + NQS * 1024;
  // kv (K, V loaded), q_full[NQS] (Q_i and its row statistics), q_empty[NQS],
  // do_full[NQS], do_empty[NQS] (dV done: dO_i and the P^T tile free), s,
  // s_consumed, dp, p, ds, kv_done (dK, dV complete), done, kv_empty (K, V no
  // longer read)
  static constexpr int B_KV = 0, B_QF = 1, B_QE = 1 + NQS, B_OF = 1 + 2 * NQS,
                       B_OE = 1 + 3 * NQS, B_S = 1 + 4 * NQS, B_SC = 2 + 4 * NQS,
                       B_DP = 3 + 4 * NQS, B_P = 4 + 4 * NQS, B_DS = 5 + 4 * NQS,
                       B_KVD = 6 + 4 * NQS, B_DONE = 7 + 4 * NQS, B_KVE = 8 + 4 * NQS,
                       NBAR = 9 + 4 * NQS;
  static constexpr int S_MISC = S_BAR + 8 * NBAR;
  static constexpr int S_META = S_MISC + 16;   // [NQS] entry index of each stage
  static constexpr int LAYOUT = S_META + 16;
  // dynamic shared memory: the layout plus as much of the 1024-byte alignment
  // slack as the per-block limit leaves (the kernel checks the actual slack)
  static constexpr int SMEM_BYTES = LAYOUT + 1024 <= 232448 ? LAYOUT + 1024 : 232448;
  static constexpr int PRODUCER = 4 * NWG, MMA = 4 * NWG + 1;  // warp indices
  static constexpr int THREADS = 128 * NWG + 64;
  static_assert(LAYOUT <= 232448, "shared memory budget");
  static_assert(NQS <= 4, "stage metadata slots");
  static_assert(NWG % 2 == 0 && D % (8 * NWG) == 0, "dK/dV columns per warpgroup");
};

template <int D, int NQS, int NWG>
__global__ void __launch_bounds__(128 * NWG + 64, 1)
    bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dk,
                  const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using C = BwdKVCfg<D, NQS, NWG>;
  constexpr int CW = C::CW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  if (smem - smem_raw + C::LAYOUT > C::SMEM_BYTES) {
    // the 1024-byte aligned layout does not fit this block's shared memory
    if (threadIdx.x == 0 && atomicCAS(p.status, 0, kErrDeviceTimeout) == 0) p.status[1] = 199;
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::S_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::S_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::S_MISC + 4);

  grid_launch_dependents();  // the dQ kernel that follows does not read our output
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Persistent CTAs: work items (key/value head, batch, key tile) ordered key
  // tile slowest (causal key tile 0, the most work, first) and dealt out in
  // snake order, one per CTA per round.
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
    // queries that see any key of [k0, k0 + BC): key j is visible to query i
    // iff j - wr <= i <= j + wl
    const int q_lo = p.wr < 0 ? 0 : max(0, I.k0 - p.wr);
    const int q_hi = p.wl < 0 ? p.N : min(p.N, min(p.N, I.k0 + C::BC) + p.wl);
    I.i_first = q_lo / C::BR;
    I.per_head = (q_hi + C::BR - 1) / C::BR - I.i_first;
    // entries: query heads of the group x query tiles in the window range, in
    // that order; with a block-sparse mask only the marked tile pairs count
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
  // computed entries of an item (whole warp)
  auto count = [&](const KVItem& I) -> int {
    if (!sparse) return I.E;
    int c = 0;
    for (int base = 0; base < I.E; base += 32)
      c += __popc(__ballot_sync(0xffffffffu, base + lane < I.E && marked(I, base + lane)));
    return c;
  };
  volatile int* meta = reinterpret_cast<volatile int*>(smem + C::S_META);
#ifdef ETA_TRACE
  const int tcta = blockIdx.x == 0 ? 0 : (blockIdx.x == 1 ? 1 : -1);
#else
  const int tcta = -1;
#endif
  (void)tcta;

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_KV), 1);
    mbar_init(BAR(C::B_KVE), 1);
    for (int s = 0; s < NQS; ++s) {
      mbar_init(BAR(C::B_QF + s), 1);
      mbar_init(BAR(C::B_QE + s), 1);
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
  // tiles) of all items so far, and the K/V and dK/dV barriers count items
  // that compute at least one entry.

  if (warp < 4 * NWG) {
    // ---------------------------------------- P^T, dS^T rows (thread j = key row j)
    const int par = warp >> 2;           // query columns [CW par, CW par + CW) of each tile
    const int j = threadIdx.x & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t st_addr = tmem + lane_base + C::T_ST + CW * par;
    const uint32_t dpt_addr = tmem + lane_base + C::T_DPT + CW * par;
    // this thread's part of its 128-byte P^T row in the 128-byte-swizzled
    // chunk holding its columns: 16-byte granules g0 .. g0 + CW/8 - 1
    uint8_t* prow = smem + C::S_P + ((CW * par) / 64) * C::CHUNK + j * 128;
    const int g0 = ((CW * par) % 64) / 8;
    const int swz = j & 7;
    // NWG = 2: this warp's P^T rows (32 rows x 128 bytes) also stage its
    // dK/dV rows for the TMA stores of the epilogue
    constexpr bool kTmaEpi = NWG == 2;
    uint8_t* stage = smem + C::S_P + par * C::CHUNK + (warp & 3) * 32 * 128;
    bool store_pending = false;  // a TMA store may still read `stage`
    bool ok = true;
    int g = 0, nkvd = 0;
    for (int r = 0; ok; ++r) {
      const KVItem I = item_of(r);
      if (!I.valid) break;
      const int n = count(I);
      const int jg = I.k0 + j;
      for (int it = 0; it < n; ++it, ++g) {
        const int stage = g % NQS;
        if (!W.wait_warp(BAR(C::B_S), g & 1, 130)) { ok = false; break; }
        // (complete already: S^T was computed from this stage) orders the reads of
        // the stage's entry index and row statistics after the producer's writes
        if (!W.wait_warp(BAR(C::B_QF + stage), (g / NQS) & 1, 134)) { ok = false; break; }
        if (j == 0) ETA_TRACE_AT(tcta, par & 1, g, 0);
        tc_fence_after();
        float pr[CW];
        tmem_load_row<CW>(st_addr, pr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_SC));  // S^T may be overwritten
        const float* lse2 =
            reinterpret_cast<const float*>(smem + C::S_STAT + stage * 1024) + CW * par;
        const float* dlt = lse2 + 128;
        const int ig0 = qtile_of(I, meta[stage]) * C::BR + CW * par;
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
        // the dV MMA of the previous tile must be done reading P^T (and the
        // epilogue's TMA stores with the staging rows): dV(g-1) completing is
        // what frees entry g-1's dO stage, whose next release needs P^T of a
        // later entry, so its parity cannot alias
        if (g > 0 && !W.wait_warp(BAR(C::B_OE + (g - 1) % NQS), ((g - 1) / NQS) & 1, 133)) {
          ok = false;
          break;
        }
        if (kTmaEpi && store_pending) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          store_pending = false;
        }
#pragma unroll
        for (int gr = 0; gr < CW / 8; ++gr) {
          const uint4 w = make_uint4(pack_bf16x2(pr[8 * gr + 0], pr[8 * gr + 1]),
                                     pack_bf16x2(pr[8 * gr + 2], pr[8 * gr + 3]),
                                     pack_bf16x2(pr[8 * gr + 4], pr[8 * gr + 5]),
                                     pack_bf16x2(pr[8 * gr + 6], pr[8 * gr + 7]));
          *reinterpret_cast<uint4*>(prow + (((g0 + gr) ^ swz) << 4)) = w;
        }
        fence_proxy_async_smem();  // generic-proxy smem writes -> tensor core reads
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_P));
        if (j == 0) ETA_TRACE_AT(tcta, par & 1, g, 1);
        if (!W.wait_warp(BAR(C::B_DP), g & 1, 131)) { ok = false; break; }
        if (j == 0) ETA_TRACE_AT(tcta, par & 1, g, 2);
        tc_fence_after();
#pragma unroll
        for (int h2 = 0; h2 < CW / 32; ++h2) {
          uint32_t rd[32];
          tmem_ld32(dpt_addr + 32 * h2, rd);
          tmem_wait_ld();
          uint32_t dk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const int c = 32 * h2 + i;
            const float2 dd = *reinterpret_cast<const float2*>(dlt + c);
            const float2 gd = fsub2(make_float2(u2f(rd[i]), u2f(rd[i + 1])), dd);
            dk[i / 2] = pack_bf16x2(pr[c] * gd.x, pr[c + 1] * gd.y);
          }
          // dS^T of columns [32 h2, 32 h2 + 32) -> packed columns 16 h2 .. 16 h2 + 15
          // (already read: each half lies below the columns still to be loaded)
          tmem_st16(dpt_addr + 16 * h2, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::B_DS));
        if (j == 0) ETA_TRACE_AT(tcta, par & 1, g, 3);
      }
      if (!ok) break;
      // epilogue: the first NWG/2 warpgroups store dV, the others dK (x scale),
      // D / (NWG/2) columns each
      constexpr int NG = NWG / 2, DC = D / NG;
      const int which = par / NG, part = par % NG;
      __nv_bfloat16* row =
          which == 0 ? static_cast<__nv_bfloat16*>(p.dv) + I.b * p.dvsb + I.hk * p.dvsh +
                           static_cast<long long>(jg) * p.dvsn + DC * part
                     : static_cast<__nv_bfloat16*>(p.dk) + I.b * p.dksb + I.hk * p.dksh +
                           static_cast<long long>(jg) * p.dksn + DC * part;
      const bool valid = jg < p.N;
      if (n > 0) {
        if (!W.wait_warp(BAR(C::B_KVD), nkvd & 1, 132)) { ok = false; break; }
        ++nkvd;
        tc_fence_after();
        const uint32_t src = tmem + lane_base + (which ? C::T_DK : C::T_DV) + DC * part;
        if constexpr (kTmaEpi) {
          tmem_rows_tma_store<DC>(src, stage, which ? &tm_dk : &tm_dv, DC * part,
                                  I.k0 + (warp & 3) * 32, I.hk, I.b, which ? p.scale : 1.f);
          store_pending = true;
        } else {
          tmem_row_to_bf16<DC>(src, row, which ? p.scale : 1.f, valid);
        }
      } else if (valid) {
        // no query sees these keys: their gradients are zero
        for (int c = 0; c < DC / 8; ++c) reinterpret_cast<uint4*>(row)[c] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // the staging rows must stay untouched until the last TMA store has read them
    if (kTmaEpi && store_pending && lane == 0) bulk_wait_read_all();
    __syncwarp();
  } else if (warp == C::PRODUCER) {
    // ---------------------------------------- TMA producer (the whole warp scans
    // 32 entries at a time; lane 0 waits and issues the copies)
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
    }
    // dO_i and Q_i have their own barriers: dO_i's slot frees earlier (after
    // dV) and is refilled first; Q_i (needed first, by S^T) follows.  An
    // item's K and V are loaded (once the previous item's last S^T and dP^T
    // are done with them) before its first computed entry.
    int g = 0, m = 0, issued_q = 0, issued_do = 0;
    bool pok = true;
    for (int r = 0; pok; ++r) {
      const KVItem I = item_of(r);
      if (!I.valid) break;
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
              if (m > 0 && !W.wait(BAR(C::B_KVE), (m - 1) & 1, 145)) {
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
            const int stage = g % NQS;
            const uint32_t par_empty = ((g / NQS) & 1) ^ 1;
            const int h = head_of(I, e);
            const int ig0 = qtile_of(I, e) * C::BR;
            if (!pok) {
            } else if (!W.wait(BAR(C::B_OE + stage), par_empty, 143)) {
              pok = false;
            } else {
              const uint32_t ofull = BAR(C::B_OF + stage);
              mbar_expect_tx(ofull, C::TILE);
              for (int c = 0; c < C::NCHUNK; ++c)
                tma_load_4d_hint(sbase + C::S_DO + stage * C::TILE + c * C::CHUNK, &tm_do, ofull,
                                 c * 64, ig0, h, I.b, l2_policy_evict_last());
              issued_do = g + 1;
              if (!W.wait(BAR(C::B_QE + stage), par_empty, 140)) {
                pok = false;
              } else {
                ETA_TRACE_AT(tcta, 3, g, 0);
                meta[stage] = e;
                const uint32_t full = BAR(C::B_QF + stage);
                mbar_expect_tx(full, C::TILE + 1024);
                for (int c = 0; c < C::NCHUNK; ++c)
                  if (!((p.debug_flags & 2) && g == 1))
                    tma_load_4d_hint(sbase + C::S_Q + stage * C::TILE + c * C::CHUNK, &tm_q, full,
                                     c * 64, ig0, h, I.b, l2_policy_evict_last());
                const long long srow = static_cast<long long>(I.b * p.Hq + h) * p.Npad + ig0;
                bulk_load(sbase + C::S_STAT + stage * 1024, p.lse2 + srow, 512, full);
                bulk_load(sbase + C::S_STAT + stage * 1024 + 512, p.delta + srow, 512, full);
                issued_q = g + 1;
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
      if (m > 0) W.drain(BAR(C::B_KV), static_cast<uint32_t>(m - 1) & 1u, 141);
      for (int s = 0; s < NQS && s < issued_q; ++s) {
        const int last = s + ((issued_q - 1 - s) / NQS) * NQS;
        W.drain(BAR(C::B_QF + s), static_cast<uint32_t>(last / NQS) & 1u, 142);
      }
      for (int s = 0; s < NQS && s < issued_do; ++s) {
        const int last = s + ((issued_do - 1 - s) / NQS) * NQS;
        W.drain(BAR(C::B_OF + s), static_cast<uint32_t>(last / NQS) & 1u, 144);
      }
    }
    __syncwarp();
  } else if (warp == C::MMA) {
    // ---------------------------------------- MMA issuer (whole warp, one elected lane issues)
    constexpr uint32_t id_s = idesc_make(128, 128, 1u, false, false);  // S^T, dP^T
    constexpr uint32_t id_kv = idesc_make(128, D, 1u, false, true);    // dV, dK
    const SDesc dK = sdesc_base(sbase + C::S_K, 16, 1024);
    const SDesc dV = sdesc_base(sbase + C::S_V, 16, 1024);
    const SDesc dP = sdesc_base(sbase + C::S_P, 16, 1024);
    auto issue_s = [&](int g) -> bool {
      const int stage = g % NQS;
      if (!W.wait_warp(BAR(C::B_QF + stage), (g / NQS) & 1, 150)) return false;
      tc_fence_after();
      const SDesc dq = sdesc_base(sbase + C::S_Q + stage * C::TILE, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
        mma_ss_w(tmem + C::T_ST, sdesc_at(dK, off), sdesc_at(dq, off), id_s, ks > 0);
      }
      mma_commit_w(BAR(C::B_S));
      return true;
    };
    auto issue_dp = [&](int g) -> bool {
      const int stage = g % NQS;
      if (!W.wait_warp(BAR(C::B_OF + stage), (g / NQS) & 1, 156)) return false;
      tc_fence_after();
      const SDesc ddo = sdesc_base(sbase + C::S_DO + stage * C::TILE, 16, 1024);
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
      if (!W.wait_warp(BAR(C::B_KV), nkv & 1, 151)) { ok = false; break; }
      ++nkv;
      // the item's first S^T overwrites S^T of the previous item's last entry
      if (g > 0 && !W.wait_warp(BAR(C::B_SC), (g - 1) & 1, 157)) { ok = false; break; }
      if (!issue_s(g) || !issue_dp(g)) { ok = false; break; }
      if (n == 1) mma_commit_w(BAR(C::B_KVE));  // K and V are not read again
      for (int it = 0; it < n; ++it, ++g) {
        const int stage = g % NQS;
        const uint32_t acc0 = it > 0 ? 1u : 0u;
        ETA_TRACE_AT(tcta, 2, g, 0);
        // S^T of the next tile once the elementwise warps have loaded this one
        if (it + 1 < n) {
          if (!W.wait_warp(BAR(C::B_SC), g & 1, 155)) { ok = false; break; }
          ETA_TRACE_AT(tcta, 3, g, 1);
          if (!issue_s(g + 1)) { ok = false; break; }
        }
        ETA_TRACE_AT(tcta, 2, g, 1);
        // dV += P^T dO_i: A = P^T (K-major shared memory), B = dO_i (MN-major)
        if (!W.wait_warp(BAR(C::B_P), g & 1, 152)) { ok = false; break; }
        ETA_TRACE_AT(tcta, 2, g, 2);
        tc_fence_after();
        const SDesc ddo = sdesc_base(sbase + C::S_DO + stage * C::TILE, C::CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss_w(tmem + C::T_DV, sdesc_at(dP, (ks >> 2) * C::CHUNK + (ks & 3) * 32),
                   sdesc_at(ddo, ks * 2048), id_kv, ks > 0 ? 1u : acc0);
        mma_commit_w(BAR(C::B_OE + stage));  // dO_i and P^T are not read again
        ETA_TRACE_AT(tcta, 3, g, 2);
        // dK += dS^T Q_i with dS^T read from TMEM
        if (!W.wait_warp(BAR(C::B_DS), g & 1, 153)) { ok = false; break; }
        ETA_TRACE_AT(tcta, 2, g, 3);
        tc_fence_after();
        const SDesc dq = sdesc_base(sbase + C::S_Q + stage * C::TILE, C::CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_w(tmem + C::T_DK, tmem + C::T_DPT + packed_col<CW>(ks), sdesc_at(dq, ks * 2048),
                   id_kv, ks > 0 ? 1u : acc0);
        mma_commit_w(BAR(C::B_QE + stage));  // Q_i (and its statistics) are not read again
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
    W.drain(BAR(C::B_DONE), 0, 154);
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
