// dQ from stored dS tiles (head dimension 128).
//
// The seven-product backward recomputes S = Q K_j^T and dP = dO V_j^T in its
// row-parallel dQ kernel only to rebuild dS, which the column-parallel dK/dV
// kernel has already computed (as dS^T, for dK += dS^T Q_i).  When the
// caller's workspace holds them, the dK/dV kernel also writes every visible
// tile's dS^T to global memory and the kernel here forms
//
//     dQ_i = scale * sum over visible key tiles j of dS_ij K_j,
//
// one product per tile pair instead of three; S, P and dP are not
// recomputed.  The sum runs over j in increasing order inside one CTA, so the
// results stay bitwise reproducible (no atomics).  This is the backward's
// "scratch for partial sums" variant that the FlashAttention (Metal Port)
// README, Documentation section, sets beside the atomic-free seven-product
// form; here the scratch holds dS rather than dQ partials.
//
// Layout of a stored tile (32 KB, bf16): the shared-memory image of dS_ij as
// an MN-major A operand without swizzling (M = 128 queries, K = 128 keys):
// 16 query groups of 8 (2 KB each, in query order), in each group 128 keys'
// 16-byte rows (8 queries' values of one key) in key order.  A core matrix
// (8 queries x 8 keys) is then 128 contiguous bytes, 128 bytes from its
// neighbour along K and 2 KB from its neighbour along M, and one bulk copy
// lands the tile ready for tcgen05.mma.  The dK/dV kernel's thread for key j
// holds 64 queries' dS^T values of that key: its 16-byte units go to groups
// 8 g .. 8 g + 7 at row j, so that a warp's 32 keys fill 512 contiguous bytes
// per store instruction.
//
// Tiles are addressed per (batch, query head): for the causal mask the
// visible tiles of query tile i are key tiles [0, i], at slot i (i + 1) / 2 + j;
// for other windows (and no mask) query tile i has a band of ds_w slots,
// slot i ds_w + j - j_lo(i).  Block-sparse masks use the window's slots and
// leave unmarked ones unwritten and unread.
#pragma once

#include <algorithm>

#include "bwd_split.cuh"

namespace eta {

constexpr int kDsTileBytes = 128 * 128 * 2;
// No stored-dS scratch beyond this size: the seven-product path runs instead.
constexpr size_t kDsMaxBytes = size_t(4) << 30;

// Slot of the stored tile (query tile i, key tile j) of (batch b, query head h).
__host__ __device__ __forceinline__ long long ds_slot(const BwdParams& p, int b, int h, int i,
                                                      int j) {
  const long long head = static_cast<long long>(b) * p.Hq + h;
  if (p.ds_tri) return head * p.ds_head + static_cast<long long>(i) * (i + 1) / 2 + j;
  const int jlo = key_tiles(128 * i, p.N, p.wl, p.wr, 128).x;
  return head * p.ds_head + static_cast<long long>(i) * p.ds_w + (j - jlo);
}

// Slot layout for N keys under the window (wl, wr) (-1 = unbounded, already
// normalised: a side >= N is -1): causal triangle or band width, tiles per head.
inline void ds_layout(int N, int wl, int wr, int* tri, int* w, long long* per_head) {
  const int nt = (N + 127) / 128;
  if (wl < 0 && wr == 0) {
    *tri = 1;
    *w = 0;
    *per_head = static_cast<long long>(nt) * (nt + 1) / 2;
    return;
  }
  int wmax = 0;
  for (int i = 0; i < nt; ++i) {
    const int2 r = key_tiles(128 * i, N, wl, wr, 128);
    wmax = std::max(wmax, r.y - r.x);
  }
  *tri = 0;
  *w = wmax;
  *per_head = static_cast<long long>(nt) * wmax;
}

// Bytes of stored dS tiles for these sizes and window (0 where the path does
// not apply: head dimension other than 128, or more than kDsMaxBytes).
inline size_t ds_bytes(int B, int Hq, int N, int D, int wl, int wr) {
  if (D != 128 || B < 1 || Hq < 1 || N < 1) return 0;
  int tri = 0, w = 0;
  long long per_head = 0;
  ds_layout(N, wl, wr, &tri, &w, &per_head);
  const size_t bytes = static_cast<size_t>(B) * Hq * per_head * kDsTileBytes;
  return bytes <= kDsMaxBytes ? bytes : 0;
}

// Offset of the stored tiles in the workspace (after the row statistics).
inline size_t ds_offset(int B, int Hq, int N, int D) {
  return round_up(bwd_workspace_bytes(B, Hq, N, D), 65536);
}

template <int NS_>
struct BwdDqsCfg {
  static constexpr int NS = NS_;              // stages of (dS tile, K tile)
  static constexpr int CHUNK = 128 * 128;     // 64 columns x 128 rows of bf16
  static constexpr int TILE = 2 * CHUNK;      // 32 KB
  static constexpr int S_DS = 0;              // [NS] dS tiles
  static constexpr int S_K = NS * TILE;       // [NS] K tiles
  static constexpr int S_EPI = 2 * NS * TILE; // epilogue staging: 8 KB per warp
  static constexpr int S_BAR = S_EPI + 4 * 8192;
  // full[NS] (dS and K landed), empty[NS] (their product is done),
  // acc_full[2] (an item's dQ is complete), acc_empty[2] (the epilogue has
  // read it), done (the MMA warp's last commit)
  static constexpr int B_F = 0, B_E = NS, B_AF = 2 * NS, B_AE = 2 * NS + 2, B_DONE = 2 * NS + 4,
                       NBAR = 2 * NS + 5;
  static constexpr int S_MISC = S_BAR + 8 * NBAR;
  static constexpr int SMEM_BYTES = S_MISC + 16 + 1024;
  static constexpr int EPI_WARPS = 4, PRODUCER = 4, MMA = 5, THREADS = 192;
  static constexpr int TMEM_COLS = 256;       // dQ[2] (fp32, 128 query lanes x 128 columns)
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// One work item of the stored-dS dQ kernel: a 128-row query tile of one
// (batch, query head), numbered query tile slowest from the last (the most
// key tiles under the causal mask) to the first.
struct DqsItem {
  int b, h, qb, jlo, jhi;
};

template <int NS>
__global__ void __launch_bounds__(192, 1)
    bwd_dqs_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_dq,
                   const BwdParams p) {
  using C = BwdDqsCfg<NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::S_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::S_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::S_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Persistent CTAs over the query tiles, dealt out in snake order (as the
  // dK/dV kernel's items): the longest first, and per CTA the sums even out.
  const int nqt = (p.N + 127) / 128;
  const int items = nqt * p.Hq * p.B;
  const bool sparse = p.bmask != nullptr;
  auto item_of = [&](int r, DqsItem& I) -> bool {
    const int w = snake_item(r, blockIdx.x, gridDim.x, items);
    if (w < 0) return false;
    I.qb = nqt - 1 - w / (p.Hq * p.B);
    I.b = (w / p.Hq) % p.B;
    I.h = w % p.Hq;
    const int2 kr = key_tiles(I.qb * 128, p.N, p.wl, p.wr, 128);
    I.jlo = kr.x;
    I.jhi = kr.y;
    return true;
  };
  // block-sparse: whether key tile j is computed for the item (any lane)
  auto marked = [&](const DqsItem& I, int j) -> bool {
    return p.bmask[((static_cast<long long>(I.b) * p.Hq + I.h) * p.nt + I.qb) * p.nt + j] != 0;
  };
  // number of computed key tiles of the item (whole warp)
  auto count = [&](const DqsItem& I) -> int {
    if (!sparse) return I.jhi - I.jlo;
    int c = 0;
    for (int base = I.jlo; base < I.jhi; base += 32)
      c += __popc(__ballot_sync(0xffffffffu, base + lane < I.jhi && marked(I, base + lane)));
    return c;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(BAR(C::B_F + s), 1);
      mbar_init(BAR(C::B_E + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(BAR(C::B_AF + a), 1);
      mbar_init(BAR(C::B_AE + a), C::EPI_WARPS);
    }
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
  // Items with at least one computed key tile take the accumulators in
  // turn: the a-th such item of this CTA uses dQ[a % 2].

  if (warp < C::EPI_WARPS) {
    // ---------------------------------------- epilogue (thread r = query row r of the item)
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    uint8_t* stage = smem + C::S_EPI + warp * 8192;
    int a = 0;
    DqsItem I;
    for (int r = 0; item_of(r, I); ++r) {
      const int n = count(I);
      const int qrow = I.qb * 128 + (threadIdx.x & 127);
      if (n == 0) {
        // no key tile is computed for this query tile: dQ = 0
        if (qrow < p.N) {
          __nv_bfloat16* row = static_cast<__nv_bfloat16*>(p.dq) + I.b * p.dqsb + I.h * p.dqsh +
                               static_cast<long long>(qrow) * p.dqsn;
          for (int c = 0; c < 16; ++c)
            reinterpret_cast<uint4*>(row)[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      const int buf = a & 1;
      if (!W.wait_warp(BAR(C::B_AF + buf), (a >> 1) & 1, 302)) break;
      tc_fence_after();
      // the previous item's stores have read the staging region
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      // dQ x scale in bf16 through TMA stores ({64, 32} boxes, 4 KB each)
      tmem_rows_tma_store<128>(tmem + lane_base + 128 * buf, stage, &tm_dq, 0,
                               I.qb * 128 + warp * 32, I.h, I.b, p.scale, 4096u);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_AE + buf));  // dQ[buf] may be overwritten
      ++a;
    }
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
  } else if (warp == C::PRODUCER) {
    // ---------------------------------------- loads: dS_ij (one bulk copy), K_j (two boxes)
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      // The dS tiles are written by the dK/dV kernel this grid follows
      // (programmatic dependent launch): wait for its completion before the
      // first read.  Every CTA waits, so this grid's completion implies the
      // dK/dV kernel's, and later work in the stream is ordered after both.
      grid_dependency_wait();
    }
    __syncwarp();
    // dS is read once (L2 evict first); K_j by every query tile of the head
    // (evict last)
    const uint64_t pol_once = l2_policy_evict_first(), pol_k = l2_policy_evict_last();
    int u = 0;  // loads issued, over all items
    bool pok = true;
    DqsItem I;
    for (int r = 0; pok && item_of(r, I); ++r) {
      for (int base = I.jlo; pok && base < I.jhi; base += 32) {
        uint32_t pend = __ballot_sync(0xffffffffu, base + lane < I.jhi &&
                                                       (!sparse || marked(I, base + lane)));
        while (pend != 0u) {
          const int j = base + __ffs(pend) - 1;
          pend &= pend - 1u;
          if (lane == 0) {
            const int s = u % NS;
            if (!W.wait(BAR(C::B_E + s), (static_cast<uint32_t>(u / NS) & 1u) ^ 1u, 310)) {
              pok = false;
            } else {
              const uint32_t full = BAR(C::B_F + s);
              mbar_expect_tx(full, 2 * C::TILE);
              bulk_load_hint(sbase + C::S_DS + s * C::TILE,
                             p.ds + ds_slot(p, I.b, I.h, I.qb, j) * kDsTileBytes, C::TILE, full,
                             pol_once);
              for (int c = 0; c < 2; ++c)
                tma_load_4d_hint(sbase + C::S_K + s * C::TILE + c * C::CHUNK, &tm_k, full, c * 64,
                                 128 * j, I.h / p.group, I.b, pol_k);
            }
          }
          pok = __shfl_sync(0xffffffffu, pok, 0);
          if (!pok) break;
          ++u;
        }
      }
    }
    if (lane == 0) {
      for (int s = 0; s < NS && s < u; ++s) {
        const int last = s + ((u - 1 - s) / NS) * NS;
        W.drain(BAR(C::B_F + s), static_cast<uint32_t>(last / NS) & 1u, 311);
      }
    }
    __syncwarp();
  } else if (warp == C::MMA) {
    // ---------------------------------------- dQ += dS_ij K_j (whole warp, one elected lane issues)
    // A = dS (M = queries, MN-major, no swizzle: the stored image; core
    // matrices 2 KB apart along M, 128 B along K, 256 B per step of 16 keys),
    // B = K_j (N = D, MN-major, 128-byte swizzle), K = 128 keys in 8 steps
    constexpr uint32_t id_q = idesc_make(128, 128, 1u, true, true);
    bool ok = true;
    int u = 0, a = 0;
    DqsItem I;
    for (int r = 0; ok && item_of(r, I); ++r) {
      const int n = count(I);
      if (n == 0) continue;
      const int buf = a & 1;
      // the epilogue has read this accumulator's previous item
      if (!W.wait_warp(BAR(C::B_AE + buf), ((a >> 1) & 1) ^ 1, 322)) { ok = false; break; }
      tc_fence_after();
      const uint32_t acc = tmem + 128 * buf;
      for (int t = 0; t < n; ++t, ++u) {
        const int s = u % NS;
        if (!W.wait_warp(BAR(C::B_F + s), static_cast<uint32_t>(u / NS) & 1u, 320)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const SDesc da = sdesc_base_plain(sbase + C::S_DS + s * C::TILE, 128, 2048);
        const SDesc dk = sdesc_base(sbase + C::S_K + s * C::TILE, C::CHUNK, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss_w(acc, sdesc_at(da, ks * 256), sdesc_at(dk, ks * 2048), id_q,
                   (t > 0 || ks > 0) ? 1u : 0u);
        mma_commit_w(BAR(C::B_E + s));  // the stage may be refilled
      }
      if (!ok) break;
      mma_commit_w(BAR(C::B_AF + buf));  // this item's dQ is complete
      ++a;
    }
    mma_commit_w(BAR(C::B_DONE));
    W.drain(BAR(C::B_DONE), 0, 321);
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
