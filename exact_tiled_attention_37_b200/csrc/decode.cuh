// Decode (split-KV) attention over a paged key/value cache for sm_100a.
//
// The Sq newest tokens of each sequence attend to its cached keys, which
// live in 128-row pages of a shared pool (FlashAttention entity page:
// FlashPrefill V2 and vLLM findings, paged KV cache; the split-KV / decode
// step with an lse merge).  Key t of sequence b is row t % 128 of page
// block_table[b][t / 128]; query token i sits at position seqlens[b] - Sq + i
// (causal: it sees keys at positions <= its own).
//
//  * decode_kernel: one CTA per (KV split, key/value head, sequence).  The
//    M = 128 rows of its single query tile are the G query heads of the
//    group x the Sq tokens (row g * Sq + i; rows past G * Sq are zero
//    padding).  It streams its range of pages through a K/V ring (TMA, one
//    page per slot), computes S = Q K^T into a double-buffered TMEM tile,
//    the online softmax (one row per thread), and O += P V in TMEM, and
//    writes this split's normalised partial O (fp32) and its logsumexp.
//  * decode_combine_kernel: per query row, merges the splits' partials:
//    lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s (bf16).
#pragma once

#include <cuda_runtime.h>

#include "fwd.cuh"
#include "ptx.cuh"

namespace eta {

struct DecodeParams {
  const void* q;           // [B, Hq, Sq, D] bf16, unit stride on D
  long long qsb, qsh, qsn;
  void* o;                 // [B, Hq, Sq, D] bf16
  long long osb, osh, osn;
  float* lse;              // [B, Hq, Sq] fp32 contiguous
  const int* block_table;  // [B][max_pages]
  const int* seqlens;      // [B]
  float* part_o;           // [B, Hq, Sq, splits, D] fp32 (workspace)
  float* part_lse;         // [B, Hq, Sq, splits] fp32 (workspace)
  int B, Hq, Hkv, Sq, group, max_pages, splits, pages_per_split, causal;
  float scale, c;          // c = scale * log2(e)
  int* status;
  unsigned long long wait_limit_ns;
};

template <int D, int NS>
struct DecodeCfg {
  static constexpr int ROWB = D * 2;
  static constexpr int NCHUNK = ROWB / 128;
  static constexpr int CHUNK = 128 * 128;      // bytes of one 64-column chunk of a 128-row tile
  static constexpr int TILE = 128 * ROWB;
  static constexpr int QK_STEPS = ROWB / 32;
  static constexpr int PV_STEPS = 128 / 16;
  static constexpr int S_COL = 0;              // S buffers at 0 and 128
  static constexpr int O_COL = 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_KV = TILE;         // [NS] K / V pages, alternating
  static constexpr int SMEM_BAR = SMEM_KV + NS * TILE;
  // q_full (4 warps), kv_full[NS], kv_empty[NS], s_full[2], p_full[2], pv_done, o_full, done
  static constexpr int BAR_Q = 0, BAR_KVF = 1, BAR_KVE = 1 + NS, BAR_S = 1 + 2 * NS,
                       BAR_P = 3 + 2 * NS, BAR_PV = 5 + 2 * NS, BAR_O = 6 + 2 * NS,
                       BAR_DONE = 7 + 2 * NS, NBAR = 8 + 2 * NS;
  static constexpr int SMEM_MISC = SMEM_BAR + 8 * NBAR;
  static constexpr int SMEM_BYTES = SMEM_MISC + 16 + 1024;
  static constexpr int THREADS = 192;          // 4 softmax warps, producer, MMA
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int D, int NS>
__global__ void __launch_bounds__(192, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const DecodeParams p) {
  using C = DecodeCfg<D, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::SMEM_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  // The sequence length, clamped to [0, 128 max_pages] (what its block-table
  // row can hold): keys and query positions both follow the clamped length.
  const int L = static_cast<int>(
      min(static_cast<long long>(max(p.seqlens[b], 0)), 128ll * p.max_pages));
  const int npages = (L + 127) / 128;  // pages of this sequence
  const int pg0 = split * p.pages_per_split;
  const int n = max(0, min(npages, pg0 + p.pages_per_split) - pg0);  // pages of this CTA
  const int M = p.group * p.Sq;  // real query rows

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::BAR_Q), 4);
    for (int s = 0; s < NS; ++s) {
      mbar_init(BAR(C::BAR_KVF + s), 1);
      mbar_init(BAR(C::BAR_KVE + s), 1);
    }
    mbar_init(BAR(C::BAR_S + 0), 1);
    mbar_init(BAR(C::BAR_S + 1), 1);
    mbar_init(BAR(C::BAR_P + 0), 4);
    mbar_init(BAR(C::BAR_P + 1), 4);
    mbar_init(BAR(C::BAR_PV), 1);
    mbar_init(BAR(C::BAR_O), 1);
    mbar_init(BAR(C::BAR_DONE), 1);
    *abort_flag = 0u;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, p.status, p.wait_limit_ns};

  if (warp < 4) {
    // ------------------------------------------------ query rows: load, softmax, epilogue
    const int r = threadIdx.x;            // row of the query tile == TMEM lane
    const bool real = r < M;
    const int g = real ? r / p.Sq : 0, i = real ? r % p.Sq : 0;
    const int h = hk * p.group + g;
    const int pos = L - p.Sq + i;         // this token's position in its sequence
    // Q row -> 128-byte-swizzled K-major rows of the tile (zeros past M)
    {
      const uint4* src = reinterpret_cast<const uint4*>(
          static_cast<const __nv_bfloat16*>(p.q) + b * p.qsb + h * p.qsh +
          static_cast<long long>(i) * p.qsn);
#pragma unroll
      for (int gi = 0; gi < D / 8; ++gi) {
        const uint4 v = real ? src[gi] : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(smem + C::SMEM_Q + (gi >> 3) * C::CHUNK + r * 128 +
                                  (((gi & 7) ^ (r & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::BAR_Q));
    }
    const bool warp_real = 32 * warp < M;  // warps with no real row skip the arithmetic
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t o_addr = tmem + lane_base + C::O_COL;
    // visible keys of this row: [0, kend)
    const int kend = (p.causal && real) ? max(0, min(L, pos + 1)) : L;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int buf = j & 1;
      const uint32_t s_addr = tmem + lane_base + C::S_COL + 128 * buf;
      if (!W.wait_warp(BAR(C::BAR_S + buf), (j >> 1) & 1, 210)) { ok = false; break; }
      if (warp_real) {
        tc_fence_after();
        float s[128];
        tmem_load_row<128>(s_addr, s);
        const int kbase = 128 * (pg0 + j);
        apply_mask<128>(s, make_int2(0, kend - kbase));
        float alpha;
        const bool rescaled = online_softmax_step<128, 0>(s, p.c, m, l, alpha);
        tmem_store_p<128, false>(s_addr, s);
        if (rescaled && j > 0) {
          // O must hold every P V product up to page j-1 before it is rescaled
          if (!W.wait_warp(BAR(C::BAR_PV), (j - 1) & 1, 211)) { ok = false; break; }
          tc_fence_after();
          tmem_scale_row<D>(o_addr, alpha);
        }
        tmem_wait_st();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::BAR_P + (j & 1)));
    }
    // this split's partial result: O / l (fp32) and lse = m * scale + ln l
    const long long prow = (static_cast<long long>(b * p.Hq + h) * p.Sq + i) * p.splits + split;
    if (ok && n > 0 && warp_real && W.wait_warp(BAR(C::BAR_O), 0, 212)) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      float* dst = p.part_o + prow * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(o_addr + 32 * c, rr);
        tmem_wait_ld();
        if (real) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            reinterpret_cast<float4*>(dst + 32 * c)[v] =
                make_float4(u2f(rr[4 * v]) * inv_l, u2f(rr[4 * v + 1]) * inv_l,
                            u2f(rr[4 * v + 2]) * inv_l, u2f(rr[4 * v + 3]) * inv_l);
        }
      }
      if (real) p.part_lse[prow] = l > 0.f ? m * p.scale + logf(l) : -INFINITY;
    } else if (ok && n == 0 && real) {
      // no page in this split: an empty partial
      p.part_lse[prow] = -INFINITY;
      for (int c = 0; c < D / 4; ++c)
        reinterpret_cast<float4*>(p.part_o + prow * D)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else if (warp == 4) {
    // ------------------------------------------------ TMA producer (K and V pages)
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int* table = p.block_table + static_cast<long long>(b) * p.max_pages;
      int it = 0;
      for (int j = 0; j < n && !W.aborted(); ++j) {
        const int page = table[pg0 + j];
        for (int kv = 0; kv < 2; ++kv, ++it) {
          const int slot = it % NS;
          const uint32_t ph = static_cast<uint32_t>(it / NS) & 1u;
          if (!W.wait(BAR(C::BAR_KVE + slot), ph ^ 1u, 230)) break;
          mbar_expect_tx(BAR(C::BAR_KVF + slot), C::TILE);
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_4d(sbase + C::SMEM_KV + slot * C::TILE + c * C::CHUNK, kv ? &tm_v : &tm_k,
                        BAR(C::BAR_KVF + slot), c * 64, hk, 0, page);
        }
      }
      const int issued = it;
      for (int s = 0; s < NS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / NS) * NS;
        W.drain(BAR(C::BAR_KVF + s), static_cast<uint32_t>(last / NS) & 1u, 232);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_make(128, 128, 1u, false, false);
      constexpr uint32_t idesc_o = idesc_make(128, D, 1u, false, true);
      auto kslot = [&](int j) { return (2 * j) % NS; };
      auto kph = [&](int j) { return static_cast<uint32_t>((2 * j) / NS) & 1u; };
      auto vslot = [&](int j) { return (2 * j + 1) % NS; };
      auto vph = [&](int j) { return static_cast<uint32_t>((2 * j + 1) / NS) & 1u; };
      const SDesc qa = sdesc_base(sbase + C::SMEM_Q, 16, 1024);
      auto issue_s = [&](int buf, int slot) {
        const SDesc kb = sdesc_base(sbase + C::SMEM_KV + slot * C::TILE, 16, 1024);
        const uint32_t d = tmem + C::S_COL + 128 * buf;
#pragma unroll
        for (int ks = 0; ks < C::QK_STEPS; ++ks) {
          const uint32_t off = (ks >> 2) * C::CHUNK + (ks & 3) * 32;
          mma_ss<false>(d, sdesc_at(qa, off), sdesc_at(kb, off), idesc_s, ks > 0);
        }
      };
      auto issue_pv = [&](int buf, int slot, bool acc) {
        const SDesc vb = sdesc_base(sbase + C::SMEM_KV + slot * C::TILE, C::CHUNK, 1024);
        const uint32_t a = tmem + C::S_COL + 128 * buf;
        const uint32_t acc0 = acc ? 1u : 0u;
#pragma unroll
        for (int ks = 0; ks < C::PV_STEPS; ++ks)
          mma_ts<false>(tmem + C::O_COL, a + 8u * ks, sdesc_at(vb, ks * 16 * 128), idesc_o,
                        ks > 0 ? 1u : acc0);
      };
      bool ok = W.wait(BAR(C::BAR_Q), 0, 240);
      if (ok && n > 0) {
        ok = W.wait(BAR(C::BAR_KVF + kslot(0)), kph(0), 241);
        if (ok) {
          tc_fence_after();
          issue_s(0, kslot(0));
          mma_commit(BAR(C::BAR_S + 0));
          mma_commit(BAR(C::BAR_KVE + kslot(0)));
        }
      }
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n) {
          if (!W.wait(BAR(C::BAR_KVF + kslot(j + 1)), kph(j + 1), 242)) { ok = false; break; }
          tc_fence_after();
          issue_s((j + 1) & 1, kslot(j + 1));
          mma_commit(BAR(C::BAR_S + ((j + 1) & 1)));
          mma_commit(BAR(C::BAR_KVE + kslot(j + 1)));
        }
        if (!W.wait(BAR(C::BAR_P + (j & 1)), (j >> 1) & 1, 243)) { ok = false; break; }
        if (!W.wait(BAR(C::BAR_KVF + vslot(j)), vph(j), 244)) { ok = false; break; }
        tc_fence_after();
        issue_pv(j & 1, vslot(j), j > 0);
        mma_commit(BAR(C::BAR_PV));
        mma_commit(BAR(C::BAR_KVE + vslot(j)));
      }
      if (ok) mma_commit(BAR(C::BAR_O));
      mma_commit(BAR(C::BAR_DONE));
      W.drain(BAR(C::BAR_DONE), 0, 247);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Merge of the splits' partials: one warp per query row (b, h, i); lane x
// handles columns [D/32 x, D/32 (x + 1)).
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeParams p) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(p.B) * p.Hq * p.Sq;
  if (row >= rows) return;  // whole warps leave together
  const int i = static_cast<int>(row % p.Sq);
  const int bh = static_cast<int>(row / p.Sq);
  const int b = bh / p.Hq, h = bh % p.Hq;
  const float* ls = p.part_lse + row * p.splits;
  float mx = -INFINITY;
  for (int s = lane; s < p.splits; s += 32) mx = fmaxf(mx, ls[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (mx > -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      const float w = expf(ls[s] - mx);  // 0 for empty splits
      den += w;
      const float* os = p.part_o + (row * p.splits + s) * D + PER * lane;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] = fmaf(w, os[e], acc[e]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.o) + b * p.osb + h * p.osh +
                       static_cast<long long>(i) * p.osn + PER * lane;
#pragma unroll
  for (int e = 0; e < PER; e += 2)
    *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
  if (lane == 0) p.lse[row] = den > 0.f ? mx + logf(den) : -INFINITY;
}

}  // namespace eta
