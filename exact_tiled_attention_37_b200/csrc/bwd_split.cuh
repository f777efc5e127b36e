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
//    dP^T = V dO_i^T, P^T, dS^T, dV += P^T dO_i, dK += dS^T Q_i.
//
// Both read lse2 = lse log2(e) and Delta = rowsum(dO O) from the
// preprocess kernel.  All MMAs are M = 128, N = 128 (or D) shapes.
#pragma once

#include "bwd.cuh"
#include "fwd.cuh"

namespace eta {

// ============================================================ dQ kernel
template <int D, int NS_>
struct BwdQCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int ROWB = D * 2;
  static constexpr int NCHUNK = ROWB / 128;
  static constexpr int CHUNK = 128 * 128;
  static constexpr int TILE = 128 * ROWB;
  static constexpr int KSTEPS = ROWB / 32;      // S, dP over D
  static constexpr int NS = NS_;                // K/V ring slots (K_j, V_j alternate)
  // TMEM: S[2] (128 each; dS bf16 written back into its first 64 columns) | dP | dQ
  static constexpr int T_S = 0, T_DP = 256, T_DQ = 384, TMEM_COLS = 512;
  static constexpr int SMEM_Q = 0, SMEM_DO = TILE, SMEM_KV = 2 * TILE;
  static constexpr int SMEM_BAR = SMEM_KV + NS * TILE;
  // q_full, kv_full[NS], kv_empty[NS], s_full[2], dp_full, ds_full, dq_done, done
  static constexpr int B_Q = 0, B_KVF = 1, B_KVE = 1 + NS, B_S = 1 + 2 * NS, B_DP = 3 + 2 * NS,
                       B_DS = 4 + 2 * NS, B_DQ = 5 + 2 * NS, B_DONE = 6 + 2 * NS,
                       NBAR = 7 + 2 * NS;
  static constexpr int SMEM_MISC = SMEM_BAR + 8 * NBAR;
  static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;
  static constexpr int THREADS = 320;           // 2 warpgroups (64 key columns each) + producer + MMA
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int D, int NS>
__global__ void __launch_bounds__(320, 1)
    bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const BwdParams p) {
  using C = BwdQCfg<D, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::SMEM_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = gridDim.z - 1 - blockIdx.z;  // longest causal tiles first
  const int h = blockIdx.x, b = blockIdx.y;
  const int hk = h / p.group;
  const int q0 = qb * C::BM;
  const int2 ktr = key_tiles(q0, p.N, p.wl, p.wr, C::BN);
  const int j0 = ktr.x, n = ktr.y - ktr.x;  // key tiles j0 .. j0 + n - 1
#ifdef ETA_TRACE
  const int tcta = (blockIdx.x == 0 && blockIdx.y == 0) ? (qb == 31 ? 0 : (qb == 15 ? 1 : -1)) : -1;
#else
  const int tcta = -1;
#endif
  (void)tcta;

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_Q), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(BAR(C::B_KVF + s), 1);
      mbar_init(BAR(C::B_KVE + s), 1);
    }
    mbar_init(BAR(C::B_S + 0), 1);
    mbar_init(BAR(C::B_S + 1), 1);
    mbar_init(BAR(C::B_DP), 1);
    mbar_init(BAR(C::B_DS), 8);
    mbar_init(BAR(C::B_DQ), 1);
    mbar_init(BAR(C::B_DONE), 1);
    *abort_flag = 0u;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, p.status, p.wait_limit_ns};

  if (warp < 8) {
    // ---------------------------------------- dS rows (thread r = query row r), then dQ
    const int par = warp >> 2;             // key columns [64 par, 64 par + 64) of each tile
    const int r = threadIdx.x & 127;
    const int qrow = q0 + r;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const long long srow = static_cast<long long>(b * p.Hq + h) * p.Npad + qrow;
    const float lse2 = p.lse2[srow];       // +inf for padded rows: their P is exactly 0
    const float dlt = p.delta[srow];
    bool ok = true;
    for (int u = 0; u < n; ++u) {
      const int buf = u & 1;
      const uint32_t s_addr = tmem + lane_base + C::T_S + 128 * buf + 64 * par;
      if (!W.wait_warp(BAR(C::B_S + buf), (u >> 1) & 1, 100)) { ok = false; break; }
      if (r == 0) ETA_FTRACE_AT(tcta, par, u, 0);
      tc_fence_after();
      float s[64];
      tmem_load_row<64>(s_addr, s);
      const int2 cw = col_window(C::BN * (j0 + u) + 64 * par, qrow, p.N, p.wl, p.wr);
      const float2 c2 = make_float2(p.c, p.c), nl2 = make_float2(-lse2, -lse2);
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        const float2 x = ffma2(make_float2(s[i], s[i + 1]), c2, nl2);
        s[i] = (i < cw.x || i >= cw.y) ? 0.f : ex2(x.x);
        s[i + 1] = (i + 1 < cw.x || i + 1 >= cw.y) ? 0.f : ex2(x.y);
      }
      if (r == 0) ETA_FTRACE_AT(tcta, par, u, 1);
      if (!W.wait_warp(BAR(C::B_DP), u & 1, 101)) { ok = false; break; }
      if (r == 0) ETA_FTRACE_AT(tcta, par, u, 2);
      tc_fence_after();
      float dp[64];
      tmem_load_row<64>(tmem + lane_base + C::T_DP + 64 * par, dp);
      uint32_t pk[32];
      const float2 d2 = make_float2(dlt, dlt);
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        const float2 g = fsub2(make_float2(dp[i], dp[i + 1]), d2);
        pk[i / 2] = pack_bf16x2(s[i] * g.x, s[i + 1] * g.y);
      }
      // dS (bf16 pairs) into the first 32 of this half's 64 S columns
      tmem_st32(s_addr, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_DS));
      if (r == 0) ETA_FTRACE_AT(tcta, par, u, 3);
    }
    if (ok && W.wait_warp(BAR(C::B_DQ), 0, 102)) {
      tc_fence_after();
      // dQ * scale in bf16: warpgroup par stores columns [D/2 par, D/2 par + D/2)
      const bool valid = qrow < p.N;
      __nv_bfloat16* row = static_cast<__nv_bfloat16*>(p.dq) + b * p.dqsb + h * p.dqsh +
                           static_cast<long long>(qrow) * p.dqsn + (D / 2) * par;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + C::T_DQ + (D / 2) * par + 32 * c, rr);
        tmem_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(row + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(u2f(rr[8 * v + 0]) * p.scale, u2f(rr[8 * v + 1]) * p.scale);
            w.y = pack_bf16x2(u2f(rr[8 * v + 2]) * p.scale, u2f(rr[8 * v + 3]) * p.scale);
            w.z = pack_bf16x2(u2f(rr[8 * v + 4]) * p.scale, u2f(rr[8 * v + 5]) * p.scale);
            w.w = pack_bf16x2(u2f(rr[8 * v + 6]) * p.scale, u2f(rr[8 * v + 7]) * p.scale);
            dst[v] = w;
          }
        }
      }
    }
  } else if (warp == 8) {
    // ---------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_expect_tx(BAR(C::B_Q), 2 * C::TILE);
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d(sbase + C::SMEM_Q + c * C::CHUNK, &tm_q, BAR(C::B_Q), c * 64, q0, h, b);
        tma_load_4d(sbase + C::SMEM_DO + c * C::CHUNK, &tm_do, BAR(C::B_Q), c * 64, q0, h, b);
      }
      int it = 0;
      for (int u = 0; u < n && !W.aborted(); ++u) {
        for (int kv = 0; kv < 2; ++kv, ++it) {
          const int slot = it % C::NS;
          if (!W.wait(BAR(C::B_KVE + slot), (static_cast<uint32_t>(it / C::NS) & 1u) ^ 1u, 110)) break;
          mbar_expect_tx(BAR(C::B_KVF + slot), C::TILE);
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_4d(sbase + C::SMEM_KV + slot * C::TILE + c * C::CHUNK, kv ? &tm_v : &tm_k,
                        BAR(C::B_KVF + slot), c * 64, C::BN * (j0 + u), hk, b);
        }
      }
      const int issued = it;
      W.drain(BAR(C::B_Q), 0, 111);
      for (int s = 0; s < C::NS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / C::NS) * C::NS;
        W.drain(BAR(C::B_KVF + s), static_cast<uint32_t>(last / C::NS) & 1u, 112);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_make(128, 128, 1u, false, false);  // S, dP
      constexpr uint32_t id_q = idesc_make(128, D, 1u, false, true);     // dQ += dS K
      const SDesc dq_ = sdesc_base(sbase + C::SMEM_Q, 16, 1024);
      const SDesc ddo = sdesc_base(sbase + C::SMEM_DO, 16, 1024);
      auto kslot = [&](int u) { return (2 * u) % C::NS; };
      auto kph = [&](int u) { return static_cast<uint32_t>((2 * u) / C::NS) & 1u; };
      auto vslot = [&](int u) { return (2 * u + 1) % C::NS; };
      auto vph = [&](int u) { return static_cast<uint32_t>((2 * u + 1) / C::NS) & 1u; };
      // S(u) = Q K^T into S[u % 2]
      auto issue_s = [&](int u) -> bool {
        if (!W.wait(BAR(C::B_KVF + kslot(u)), kph(u), 120)) return false;
        tc_fence_after();
        const SDesc kb = sdesc_base(sbase + C::SMEM_KV + kslot(u) * C::TILE, 16, 1024);
        const uint32_t d = tmem + C::T_S + 128 * (u & 1);
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks) {
          const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
          mma_ss<false>(d, sdesc_at(dq_, off), sdesc_at(kb, off), id_s, ks > 0);
        }
        mma_commit(BAR(C::B_S + (u & 1)));
        return true;
      };
      // dP(u) = dO V^T
      auto issue_dp = [&](int u) -> bool {
        if (!W.wait(BAR(C::B_KVF + vslot(u)), vph(u), 121)) return false;
        tc_fence_after();
        const SDesc vb = sdesc_base(sbase + C::SMEM_KV + vslot(u) * C::TILE, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks) {
          const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
          mma_ss<false>(tmem + C::T_DP, sdesc_at(ddo, off), sdesc_at(vb, off), id_s, ks > 0);
        }
        mma_commit(BAR(C::B_DP));
        mma_commit(BAR(C::B_KVE + vslot(u)));  // V_u is not read again
        return true;
      };
      bool ok = W.wait(BAR(C::B_Q), 0, 122);
      if (ok && n > 0) ok = issue_s(0) && issue_dp(0);
      if (ok && n > 1) ok = issue_s(1);
      for (int u = 0; ok && u < n; ++u) {
        // dS(u) is in S[u % 2] and dP has been read
        if (!W.wait(BAR(C::B_DS), u & 1, 123)) { ok = false; break; }
        ETA_FTRACE_AT(tcta, 2, u, 0);
        tc_fence_after();
        // dQ += dS K_u: A = dS from TMEM (key k at column (k / 64) * 64 + (k % 64) / 2),
        // B = K_u as an MN-major operand (N = D, K = 128 keys)
        const SDesc kb = sdesc_base(sbase + C::SMEM_KV + kslot(u) * C::TILE, C::CHUNK, 1024);
        const uint32_t a = tmem + C::T_S + 128 * (u & 1);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts<false>(tmem + C::T_DQ, a + 64 * (ks >> 2) + 8 * (ks & 3), sdesc_at(kb, ks * 2048),
                        id_q, (u > 0 || ks > 0) ? 1u : 0u);
        mma_commit(BAR(C::B_KVE + kslot(u)));  // K_u is not read again
        ETA_FTRACE_AT(tcta, 2, u, 1);
        if (u + 1 < n && !issue_dp(u + 1)) { ok = false; break; }
        ETA_FTRACE_AT(tcta, 2, u, 2);
        if (u + 2 < n && !issue_s(u + 2)) { ok = false; break; }
        ETA_FTRACE_AT(tcta, 2, u, 3);
      }
      if (ok) mma_commit(BAR(C::B_DQ));
      mma_commit(BAR(C::B_DONE));
      W.drain(BAR(C::B_DONE), 0, 124);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}


// ============================================================ dK / dV kernel
// P^T goes through shared memory (the A operand of dV += P^T dO_i) so that
// S^T of the next query tile can be computed as soon as the softmax
// warpgroups have loaded S^T of this one; dS^T stays in TMEM (in the dP^T
// columns it was computed from).
template <int D, int NQS>
struct BwdKVCfg {
  static constexpr int BC = 128, BR = 128;
  static constexpr int ROWB = D * 2;
  static constexpr int NCHUNK = ROWB / 128;
  static constexpr int CHUNK = 128 * 128;
  static constexpr int TILE = 128 * ROWB;
  static constexpr int KSTEPS = ROWB / 32;
  // TMEM: S^T | dP^T (dS^T bf16 written back into its first columns) | dV | dK
  static constexpr int T_ST = 0, T_DPT = 128, T_DV = 256, T_DK = 256 + D, TMEM_COLS = 512;
  static constexpr int S_K = 0, S_V = TILE, S_Q = 2 * TILE;   // [NQS] Q tiles
  static constexpr int S_DO = S_Q + NQS * TILE;                // [NQS] dO tiles
  static constexpr int S_P = S_DO + NQS * TILE;                // P^T: 128 key rows x 128 queries bf16
  static constexpr int S_STAT = S_P + 128 * 256;               // [NQS] lse2[128], delta[128]
  static constexpr int S_BAR = S_STAT + NQS * 1024;
  // kv, q_full[NQS], q_empty[NQS], s, s_consumed, dp, p, p_empty, ds, kv_done, done
  static constexpr int B_KV = 0, B_QF = 1, B_QE = 1 + NQS, B_S = 1 + 2 * NQS, B_SC = 2 + 2 * NQS,
                       B_DP = 3 + 2 * NQS, B_P = 4 + 2 * NQS, B_PE = 5 + 2 * NQS,
                       B_DS = 6 + 2 * NQS, B_KVD = 7 + 2 * NQS, B_DONE = 8 + 2 * NQS,
                       NBAR = 9 + 2 * NQS;
  static constexpr int S_MISC = S_BAR + 8 * NBAR;
  static constexpr int LAYOUT = S_MISC + 16;
  // dynamic shared memory: the layout plus as much of the 1024-byte alignment
  // slack as the per-block limit leaves (the kernel checks the actual slack)
  static constexpr int SMEM_BYTES = LAYOUT + 1024 <= 232448 ? LAYOUT + 1024 : 232448;
  static constexpr int THREADS = 320;  // 2 warpgroups (64 query columns each) + producer + MMA
  static_assert(LAYOUT <= 232448, "shared memory budget");
};

template <int D, int NQS>
__global__ void __launch_bounds__(320, 1)
    bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  using C = BwdKVCfg<D, NQS>;
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

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.z;  // causal key tile 0 (the most work) is dispatched first
  const int hk = blockIdx.x, b = blockIdx.y;
  const int k0 = kt * C::BC;
  // queries that see any key of [k0, k0 + BC): key j is visible to query i iff
  // j - wr <= i <= j + wl
  const int q_lo = p.wr < 0 ? 0 : max(0, k0 - p.wr);
  const int q_hi = p.wl < 0 ? p.N : min(p.N, min(p.N, k0 + C::BC) + p.wl);
  const int i_first = q_lo / C::BR;
  const int per_head = (q_hi + C::BR - 1) / C::BR - i_first;
  const int n = per_head * p.group;  // iterations: query heads of the group x query tiles
  auto head_of = [&](int it) { return hk * p.group + it / per_head; };
  auto qtile_of = [&](int it) { return i_first + it % per_head; };
#ifdef ETA_TRACE
  const int tcta = (blockIdx.x == 0 && blockIdx.y == 0) ? (kt == 0 ? 0 : (kt == 16 ? 1 : -1)) : -1;
#else
  const int tcta = -1;
#endif
  (void)tcta;

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_KV), 1);
    for (int s = 0; s < NQS; ++s) {
      mbar_init(BAR(C::B_QF + s), 1);
      mbar_init(BAR(C::B_QE + s), 1);
    }
    mbar_init(BAR(C::B_S), 1);
    mbar_init(BAR(C::B_SC), 8);
    mbar_init(BAR(C::B_DP), 1);
    mbar_init(BAR(C::B_P), 8);
    mbar_init(BAR(C::B_PE), 1);
    mbar_init(BAR(C::B_DS), 8);
    mbar_init(BAR(C::B_KVD), 1);
    mbar_init(BAR(C::B_DONE), 1);
    *abort_flag = 0u;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, p.status, p.wait_limit_ns};

  if (warp < 8) {
    // ---------------------------------------- P^T, dS^T rows (thread j = key row j)
    const int par = warp >> 2;           // query columns [64 par, 64 par + 64) of each tile
    const int j = threadIdx.x & 127;
    const int jg = k0 + j;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t st_addr = tmem + lane_base + C::T_ST + 64 * par;
    const uint32_t dpt_addr = tmem + lane_base + C::T_DPT + 64 * par;
    // this thread's 128-byte row of P^T in the 128-byte-swizzled chunk of its columns
    uint8_t* prow = smem + C::S_P + par * C::CHUNK + j * 128;
    const int swz = j & 7;
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int stage = it % NQS;
      if (!W.wait_warp(BAR(C::B_S), it & 1, 130)) { ok = false; break; }
      if (j == 0) ETA_TRACE_AT(tcta, par, it, 0);
      tc_fence_after();
      float pr[64];
      tmem_load_row<64>(st_addr, pr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_SC));  // S^T may be overwritten
      const float* lse2 = reinterpret_cast<const float*>(smem + C::S_STAT + stage * 1024) + 64 * par;
      const float* dlt = lse2 + 128;
      const int ig0 = qtile_of(it) * C::BR + 64 * par;
      // window: query ig0 + i sees key jg iff jg - wr <= ig0 + i <= jg + wl
      const int ilo = p.wr < 0 ? -(1 << 30) : jg - p.wr - ig0;
      const int ihi = p.wl < 0 ? (1 << 30) : jg + p.wl - ig0;
      const float2 c2 = make_float2(p.c, p.c);
      if (ilo <= 0 && ihi >= 63) {
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          const float2 l2 = *reinterpret_cast<const float2*>(lse2 + i);
          const float2 x = ffma2(make_float2(pr[i], pr[i + 1]), c2, make_float2(-l2.x, -l2.y));
          pr[i] = ex2(x.x);
          pr[i + 1] = ex2(x.y);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          const float2 l2 = *reinterpret_cast<const float2*>(lse2 + i);
          const float2 x = ffma2(make_float2(pr[i], pr[i + 1]), c2, make_float2(-l2.x, -l2.y));
          pr[i] = (i < ilo || i > ihi) ? 0.f : ex2(x.x);
          pr[i + 1] = (i + 1 < ilo || i + 1 > ihi) ? 0.f : ex2(x.y);
        }
      }
      // the dV MMA of the previous tile must be done reading P^T
      if (!W.wait_warp(BAR(C::B_PE), (it & 1) ^ 1, 133)) { ok = false; break; }
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const uint4 w = make_uint4(pack_bf16x2(pr[8 * g + 0], pr[8 * g + 1]),
                                   pack_bf16x2(pr[8 * g + 2], pr[8 * g + 3]),
                                   pack_bf16x2(pr[8 * g + 4], pr[8 * g + 5]),
                                   pack_bf16x2(pr[8 * g + 6], pr[8 * g + 7]));
        *reinterpret_cast<uint4*>(prow + ((g ^ swz) << 4)) = w;
      }
      fence_proxy_async_smem();  // generic-proxy smem writes -> tensor core reads
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_P));
      if (j == 0) ETA_TRACE_AT(tcta, par, it, 1);
      if (!W.wait_warp(BAR(C::B_DP), it & 1, 131)) { ok = false; break; }
      if (j == 0) ETA_TRACE_AT(tcta, par, it, 2);
      tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t rd[32];
        tmem_ld32(dpt_addr + 32 * h2, rd);
        tmem_wait_ld();
        uint32_t dk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int c = 32 * h2 + i;
          const float2 dd = *reinterpret_cast<const float2*>(dlt + c);
          const float2 g = fsub2(make_float2(u2f(rd[i]), u2f(rd[i + 1])), dd);
          dk[i / 2] = pack_bf16x2(pr[c] * g.x, pr[c + 1] * g.y);
        }
        // dS^T of columns [32 h2, 32 h2 + 32) -> dP^T columns 16 h2 .. 16 h2 + 15
        // (already read: each half lies below the columns still to be loaded)
        tmem_st16(dpt_addr + 16 * h2, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_DS));
      if (j == 0) ETA_TRACE_AT(tcta, par, it, 3);
    }
    if (ok && n > 0 && W.wait_warp(BAR(C::B_KVD), 0, 132)) {
      tc_fence_after();
      // even warpgroup stores dV, odd warpgroup stores dK (x scale)
      const bool valid = jg < p.N;
      __nv_bfloat16* row =
          par == 0 ? static_cast<__nv_bfloat16*>(p.dv) + b * p.dvsb + hk * p.dvsh +
                         static_cast<long long>(jg) * p.dvsn
                   : static_cast<__nv_bfloat16*>(p.dk) + b * p.dksb + hk * p.dksh +
                         static_cast<long long>(jg) * p.dksn;
      const float mul = par ? p.scale : 1.f;
      const uint32_t col = par ? C::T_DK : C::T_DV;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + col + 32 * c, r);
        tmem_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(row + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(u2f(r[8 * v + 0]) * mul, u2f(r[8 * v + 1]) * mul);
            w.y = pack_bf16x2(u2f(r[8 * v + 2]) * mul, u2f(r[8 * v + 3]) * mul);
            w.z = pack_bf16x2(u2f(r[8 * v + 4]) * mul, u2f(r[8 * v + 5]) * mul);
            w.w = pack_bf16x2(u2f(r[8 * v + 6]) * mul, u2f(r[8 * v + 7]) * mul);
            dst[v] = w;
          }
        }
      }
    } else if (n == 0) {
      // no query sees these keys: their gradients are zero
      const bool valid = jg < p.N;
      __nv_bfloat16* row =
          par == 0 ? static_cast<__nv_bfloat16*>(p.dv) + b * p.dvsb + hk * p.dvsh +
                         static_cast<long long>(jg) * p.dvsn
                   : static_cast<__nv_bfloat16*>(p.dk) + b * p.dksb + hk * p.dksh +
                         static_cast<long long>(jg) * p.dksn;
      if (valid)
        for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(row)[c] = make_uint4(0u, 0u, 0u, 0u);
    }
  } else if (warp == 8) {
    // ---------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_expect_tx(BAR(C::B_KV), 2 * C::TILE);
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d(sbase + C::S_K + c * C::CHUNK, &tm_k, BAR(C::B_KV), c * 64, k0, hk, b);
        tma_load_4d(sbase + C::S_V + c * C::CHUNK, &tm_v, BAR(C::B_KV), c * 64, k0, hk, b);
      }
      int it = 0;
      for (; it < n; ++it) {
        const int stage = it % NQS;
        if (!W.wait(BAR(C::B_QE + stage), ((it / NQS) & 1) ^ 1, 140)) break;
        ETA_TRACE_AT(tcta, 3, it, 0);
        const int h = head_of(it);
        const int ig0 = qtile_of(it) * C::BR;
        const uint32_t full = BAR(C::B_QF + stage);
        mbar_expect_tx(full, 2 * C::TILE + 1024);
        for (int c = 0; c < C::NCHUNK; ++c) {
          tma_load_4d(sbase + C::S_Q + stage * C::TILE + c * C::CHUNK, &tm_q, full, c * 64, ig0, h, b);
          tma_load_4d(sbase + C::S_DO + stage * C::TILE + c * C::CHUNK, &tm_do, full, c * 64, ig0, h, b);
        }
        const long long srow = static_cast<long long>(b * p.Hq + h) * p.Npad + ig0;
        bulk_load(sbase + C::S_STAT + stage * 1024, p.lse2 + srow, 512, full);
        bulk_load(sbase + C::S_STAT + stage * 1024 + 512, p.delta + srow, 512, full);
      }
      W.drain(BAR(C::B_KV), 0, 141);
      const int issued = it;
      for (int s = 0; s < NQS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / NQS) * NQS;
        W.drain(BAR(C::B_QF + s), static_cast<uint32_t>(last / NQS) & 1u, 142);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_make(128, 128, 1u, false, false);  // S^T, dP^T
      constexpr uint32_t id_kv = idesc_make(128, D, 1u, false, true);    // dV, dK
      const SDesc dK = sdesc_base(sbase + C::S_K, 16, 1024);
      const SDesc dV = sdesc_base(sbase + C::S_V, 16, 1024);
      const SDesc dP = sdesc_base(sbase + C::S_P, 16, 1024);
      auto issue_s = [&](int it) -> bool {
        const int stage = it % NQS;
        if (!W.wait(BAR(C::B_QF + stage), (it / NQS) & 1, 150)) return false;
        tc_fence_after();
        const SDesc dq = sdesc_base(sbase + C::S_Q + stage * C::TILE, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks) {
          const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
          mma_ss<false>(tmem + C::T_ST, sdesc_at(dK, off), sdesc_at(dq, off), id_s, ks > 0);
        }
        mma_commit(BAR(C::B_S));
        return true;
      };
      auto issue_dp = [&](int it) {
        const int stage = it % NQS;
        const SDesc ddo = sdesc_base(sbase + C::S_DO + stage * C::TILE, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks) {
          const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
          mma_ss<false>(tmem + C::T_DPT, sdesc_at(dV, off), sdesc_at(ddo, off), id_s, ks > 0);
        }
        mma_commit(BAR(C::B_DP));
      };
      bool ok = W.wait(BAR(C::B_KV), 0, 151);
      if (ok && n > 0) {
        ok = issue_s(0);
        if (ok) issue_dp(0);
      }
      for (int it = 0; ok && it < n; ++it) {
        const int stage = it % NQS;
        const uint32_t acc0 = it > 0 ? 1u : 0u;
        ETA_TRACE_AT(tcta, 2, it, 0);
        // S^T of the next tile once the softmax has loaded this one
        if (it + 1 < n) {
          if (!W.wait(BAR(C::B_SC), it & 1, 155)) { ok = false; break; }
          if (!issue_s(it + 1)) { ok = false; break; }
        }
        ETA_TRACE_AT(tcta, 2, it, 1);
        // dV += P^T dO_i: A = P^T (K-major shared memory), B = dO_i (MN-major)
        if (!W.wait(BAR(C::B_P), it & 1, 152)) { ok = false; break; }
        ETA_TRACE_AT(tcta, 2, it, 2);
        tc_fence_after();
        const SDesc ddo = sdesc_base(sbase + C::S_DO + stage * C::TILE, C::CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss<false>(tmem + C::T_DV, sdesc_at(dP, (ks >> 2) * C::CHUNK + (ks & 3) * 32),
                        sdesc_at(ddo, ks * 2048), id_kv, ks > 0 ? 1u : acc0);
        mma_commit(BAR(C::B_PE));
        // dK += dS^T Q_i: dS^T of query column k at dP^T column 64 (k / 64) + (k % 64) / 2
        if (!W.wait(BAR(C::B_DS), it & 1, 153)) { ok = false; break; }
        ETA_TRACE_AT(tcta, 2, it, 3);
        tc_fence_after();
        const SDesc dq = sdesc_base(sbase + C::S_Q + stage * C::TILE, C::CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts<false>(tmem + C::T_DK, tmem + C::T_DPT + 64 * (ks >> 2) + 8 * (ks & 3),
                        sdesc_at(dq, ks * 2048), id_kv, ks > 0 ? 1u : acc0);
        mma_commit(BAR(C::B_QE + stage));
        if (it + 1 < n) issue_dp(it + 1);
      }
      if (ok) mma_commit(BAR(C::B_KVD));
      mma_commit(BAR(C::B_DONE));
      W.drain(BAR(C::B_DONE), 0, 154);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace eta
