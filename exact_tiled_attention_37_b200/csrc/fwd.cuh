// Forward attention kernels for sm_100a.
//
// O = softmax(scale * Q K^T [+ causal mask]) V and lse = log(sum exp(...)),
// computed tile by tile with an online softmax and deferred normalisation,
// so the N x N score matrix never leaves the SM (the tiled online softmax of
// FA1, the query-tile ownership and single final division of FA2, the staged
// ping-pong pipeline of FA3 and the load / MMA / softmax roles with a
// conditional rescale of FA4, as listed in the r/mlscaling FlashAttention-
// PyTorch post; tensor-memory accumulators and asynchronous TMA/MMA pipelines
// as in the "FlashAttention-4: Algorithm and Kernel Pipelining for Blackwell
// GPUs" finding on the FlashAttention entity page).
//
// The kernel, fwd_single_kernel: one 128-row query tile per CTA, 64-row K/V
// tiles through a TMA ring and a double-buffered S, so that S(j+1) =
// Q K_{j+1}^T runs while the row softmax works on S(j).  TMEM: S0 | S1 | O.
// At D <= 128 these take 256 columns and two CTAs share an SM (one CTA's
// loads and epilogue overlap the other's products); at D = 256 O needs 256
// columns and one CTA runs per SM.  bf16 at D = 64, 128, 256; e4m3 at D = 128.
//
// Roles (warp-specialised): a TMA producer warp, an MMA warp (one thread
// issues every tcgen05.mma), and a 128-thread softmax warpgroup in which
// thread r owns query row r (TMEM lane r).  The softmax warpgroup also
// does the correction (rescaling the O row in TMEM when its running maximum
// grows by more than 2^kRescaleLog2) and the epilogue (O / l, lse).
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace eta {

// Rescale O and l only when the running row maximum grows by more than this
// many powers of two; otherwise keep the stale maximum (results are
// identical: O and l always share the same reference maximum).
constexpr float kRescaleLog2 = 8.0f;

// Columns (of every 8) whose exponential the forward computes with the
// FMA-pipe polynomial; the rest use the MUFU ex2 unit (0: measured fastest).
#ifndef ETA_SOFT_EXP8
#define ETA_SOFT_EXP8 0
#endif
constexpr int kSoftExp8 = ETA_SOFT_EXP8;

#ifdef ETA_TRACE
// Debug builds only: clock64() timelines of two CTAs of whichever kernel
// records them ([cta][role][tile][event]); the macro is defined here so that
// every kernel header can use it, and today the backward's dQ kernel does
// (roles: elementwise warpgroups 0 and 1, MMA warp).
__device__ unsigned long long g_eta_ftrace[2][3][256][4];
#define ETA_FTRACE_AT(cta, role, it, ev)                                          \
  do {                                                                           \
    if ((cta) >= 0 && (it) < 256) g_eta_ftrace[(cta)][(role)][(it)][(ev)] = clock64(); \
  } while (0)
#else
#define ETA_FTRACE_AT(cta, role, it, ev) \
  do {                                   \
  } while (0)
#endif

struct FwdParams {
  void* o;           // [B, Hq, N, D], unit stride on D
  float* lse;        // [B, Hq, N] contiguous
  long long osb, osh, osn;
  int Hq, N, group;  // group = Hq / Hkv
  int wl, wr;        // local window: query i sees keys [i - wl, i + wr]; -1 = unbounded
  float scale;       // softmax scale (natural units)
  float c;           // scale * log2(e)
  int* status;       // device status word (4 ints)
  unsigned long long wait_limit_ns;
  int debug_flags;   // bit 0: producer skips the first V tile (timeout test)
  float o_mul;       // output multiplier (1; e4m3 inputs: v_scale / kP8Scale)
  // block-sparse tile mask [B, Hq, nt, nt] (nonzero = the 128 x 128 tile pair is
  // computed), or null; nt = ceil(N / 128) <= kMaxMaskTiles
  const uint8_t* bmask;
  int nt;
  // grid order of the kernels with one CTA per query tile: 1 = (query tiles,
  // heads, batch), a head's tiles together, for masks under which every tile
  // does about the same work; 0 = (heads, batch, query tiles), longest first
  int head_major;
};

// Longest sequence (in 128-row tiles) a block-sparse mask may describe: the
// kernels keep one bit per key tile of a query tile in shared memory.
constexpr int kMaxMaskTiles = 512;
constexpr int kMaskWords = kMaxMaskTiles / 32;

// Number of set bits of w[] below bit j.
__device__ __forceinline__ int bits_below(const uint32_t* w, int j) {
  int c = 0;
  for (int i = 0; i < (j >> 5); ++i) c += __popc(w[i]);
  if (j & 31) c += __popc(w[j >> 5] & ((1u << (j & 31)) - 1u));
  return c;
}

// Smallest set bit of w[] at or after j, or `end` (bits at or beyond `end` ignored).
__device__ __forceinline__ int next_bit(const uint32_t* w, int j, int end) {
  while (j < end) {
    const uint32_t x = w[j >> 5] >> (j & 31);
    if (x) return min(end, j + __ffs(x) - 1);
    j = (j | 31) + 1;
  }
  return end;
}

// Online-softmax update of one row over one tile of BC scores (already masked
// to -inf where not allowed).  m is the running maximum in raw score units,
// l the running sum of exp2((s - m) * c).  Converts s in place into
// p = exp2((s - m) * c).  Returns true when this warp rescaled (alpha != 1
// for some row of the warp); alpha is this row's factor for O and l.
// SOFT8 of every 8 columns take their exponential from the FMA-pipe
// polynomial instead of the MUFU unit (the two run in parallel).
// TAU: rescale only when the maximum grows by more than 2^TAU (p <= 2^TAU);
// e4m3 products need TAU = 0 (p <= 1).
template <int BC, int SOFT8, int TAU = static_cast<int>(kRescaleLog2)>
__device__ __forceinline__ bool online_softmax_step(float (&s)[BC], float c, float& m, float& l,
                                                    float& alpha) {
  static_assert(BC % 8 == 0 && SOFT8 % 2 == 0 && SOFT8 <= 8, "column pattern");
  float mx0 = fmax3(s[0], s[1], s[2]), mx1 = fmax3(s[3], s[4], s[5]);
  float mx2 = fmax3(s[6], s[7], s[8]), mx3 = fmax3(s[9], s[10], s[11]);
#pragma unroll
  for (int i = 12; i + 8 <= BC; i += 8) {
    mx0 = fmax3(mx0, s[i], s[i + 1]);
    mx1 = fmax3(mx1, s[i + 2], s[i + 3]);
    mx2 = fmax3(mx2, s[i + 4], s[i + 5]);
    mx3 = fmax3(mx3, s[i + 6], s[i + 7]);
  }
#pragma unroll
  for (int i = BC - (BC - 12) % 8; i < BC; ++i) mx0 = fmaxf(mx0, s[i]);
  const float m_new = fmaxf(m, fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)));
  // +inf when m = -inf and m_new is finite; NaN (false) when both are -inf
  const bool need = (m_new - m) * c > static_cast<float>(TAU);
  const bool warp_rescale = __any_sync(0xffffffffu, need);
  alpha = 1.f;
  if (warp_rescale) {
    alpha = (m_new == -INFINITY) ? 1.f : ex2((m - m_new) * c);
    m = m_new;
    l *= alpha;
  }
  const float nmc = (m == -INFINITY) ? 0.f : -m * c;
  const float2 c2 = make_float2(c, c), nmc2 = make_float2(nmc, nmc);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0, acc2 = acc0, acc3 = acc0;
#pragma unroll
  for (int i = 0; i < BC; i += 8) {
    float2 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = ffma2(make_float2(s[i + 2 * u], s[i + 2 * u + 1]), c2, nmc2);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float2 e;
      if (2 * u < SOFT8) {
        e = exp2_poly2(x[u]);
      } else {
        e.x = ex2(x[u].x);
        e.y = ex2(x[u].y);
      }
      s[i + 2 * u] = e.x;
      s[i + 2 * u + 1] = e.y;
    }
    acc0 = fadd2(acc0, make_float2(s[i], s[i + 1]));
    acc1 = fadd2(acc1, make_float2(s[i + 2], s[i + 3]));
    acc2 = fadd2(acc2, make_float2(s[i + 4], s[i + 5]));
    acc3 = fadd2(acc3, make_float2(s[i + 6], s[i + 7]));
  }
  const float2 a01 = fadd2(acc0, acc1), a23 = fadd2(acc2, acc3);
  const float2 a = fadd2(a01, a23);
  l += a.x + a.y;
  return warp_rescale;
}

// Writes p (BC values) back into TMEM as the A operand of the P V MMA:
// bf16 pairs packed per 32-bit column (BC/2 columns) or fp32 (BC columns).
template <int BC, bool TF32>
__device__ __forceinline__ void tmem_store_p(uint32_t taddr, const float (&p)[BC]) {
  if constexpr (TF32) {
#pragma unroll
    for (int c = 0; c < BC / 32; ++c) {
      uint32_t r[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(p[32 * c + i]);
      tmem_st32(taddr + 32 * c, r);
    }
  } else {
#pragma unroll
    for (int c = 0; c < BC / 64; ++c) {
      uint32_t r[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = pack_bf16x2(p[64 * c + 2 * i], p[64 * c + 2 * i + 1]);
      tmem_st32(taddr + 32 * c, r);
    }
    if constexpr (BC % 64 == 32) {
      uint32_t r[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) r[i] = pack_bf16x2(p[BC - 32 + 2 * i], p[BC - 32 + 2 * i + 1]);
      tmem_st16(taddr + BC / 2 - 16, r);
    }
  }
}

// e4m3 P for the kind::f8f6f4 P V product, as two terms so that P keeps about
// 8 significant bits (one e4m3 term has 4): x = p * kP8Scale (p <= 2^kP8Tau,
// so x <= 256, inside e4m3's range; the scale keeps small probabilities out of
// e4m3's subnormals), hi = e4m3(x), lo = e4m3(x - hi) (the residual, formed
// in fp16, which holds both exactly enough).  hi goes to the first BC/4
// columns, lo to the next BC/4, four values per 32-bit column.
// e4m3 builds rescale when the row maximum grows by more than 2^kP8Tau, so
// p <= 2^kP8Tau and p * kP8Scale <= 256 (e4m3's largest finite value is 448).
// Measured on B200: 2^3 runs 16 % faster than 2^0 (fewer rescales) with
// max|dO|/max|O| 2.2e-3 against 2.2e-3 (the tolerance is 2e-2).
constexpr int kP8Tau = 3;
constexpr float kP8Scale = 256.f / static_cast<float>(1 << kP8Tau);
template <int BC>
__device__ __forceinline__ void tmem_store_p8(uint32_t taddr, const float (&p)[BC]) {
  static_assert(BC == 128 || BC == 64, "32 or 16 columns per term");
  uint32_t hi[BC / 4], lo[BC / 4];
#pragma unroll
  for (int i = 0; i < BC / 4; ++i) {
    uint32_t hw = 0u, lw = 0u;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float2 x = make_float2(p[4 * i + 2 * k] * kP8Scale, p[4 * i + 2 * k + 1] * kP8Scale);
      const __nv_fp8x2_storage_t h = __nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3);
      const __half2 hf = __half2(__nv_cvt_fp8x2_to_halfraw2(h, __NV_E4M3));
      const __half2 r = __hsub2(__float22half2_rn(x), hf);
      const __nv_fp8x2_storage_t l =
          __nv_cvt_halfraw2_to_fp8x2(static_cast<__half2_raw>(r), __NV_SATFINITE, __NV_E4M3);
      hw |= static_cast<uint32_t>(h) << (16 * k);
      lw |= static_cast<uint32_t>(l) << (16 * k);
    }
    hi[i] = hw;
    lo[i] = lw;
  }
  if constexpr (BC == 128) {
    tmem_st32(taddr, hi);
    tmem_st32(taddr + BC / 4, lo);
  } else {
    tmem_st16(taddr, hi);
    tmem_st16(taddr + BC / 4, lo);
  }
}

// Multiplies DC fp32 TMEM columns of this lane by alpha (the correction step).
template <int DC>
__device__ __forceinline__ void tmem_scale_row(uint32_t taddr, float alpha) {
#pragma unroll 1
  for (int c = 0; c < DC / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + 32 * c, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(u2f(r[i]) * alpha);
    tmem_st32(taddr + 32 * c, r);
  }
}

// Epilogue of a row whose query tile computed no key tile: O = 0, lse = -inf.
template <typename T, int D>
__device__ __forceinline__ void store_empty_row(const FwdParams& p, int b, int h, int qrow) {
  if (qrow >= p.N) return;
  char* row = static_cast<char*>(p.o) +
              (static_cast<long long>(b) * p.osb + static_cast<long long>(h) * p.osh +
               static_cast<long long>(qrow) * p.osn) *
                  static_cast<long long>(sizeof(T));
  for (int i = 0; i < D * static_cast<int>(sizeof(T)) / 16; ++i)
    reinterpret_cast<uint4*>(row)[i] = make_uint4(0u, 0u, 0u, 0u);
  p.lse[(static_cast<long long>(b) * p.Hq + h) * p.N + qrow] = -INFINITY;
}

// Keys [lo, hi) that query rows [qs, qe) may see under the window (wl, wr)
// (-1 = unbounded; the causal mask is (-1, 0)), clipped to [0, N).
__host__ __device__ __forceinline__ int2 window_keys(int qs, int qe, int N, int wl, int wr) {
  const int lo = wl < 0 ? 0 : max(0, qs - wl);
  const int hi = wr < 0 ? N : min(N, qe + wr);
  return make_int2(lo, hi);
}

// Visible columns [lo, hi) of one query row in the key tile starting at kbase.
__device__ __forceinline__ int2 col_window(int kbase, int qrow, int N, int wl, int wr) {
  const int lo = wl < 0 ? 0 : qrow - wl - kbase;
  const int hi = min(N, wr < 0 ? N : qrow + wr + 1) - kbase;
  return make_int2(lo, hi);
}

template <int BC>
__device__ __forceinline__ void apply_mask(float (&s)[BC], int2 cw) {
  if (cw.x > 0 || cw.y < BC) {
#pragma unroll
    for (int i = 0; i < BC; ++i)
      if (i < cw.x || i >= cw.y) s[i] = -INFINITY;
  }
}

// Key-tile range [j_lo, j_hi) of a 128-row query tile starting at qs (empty
// when the tile lies past N).
__host__ __device__ __forceinline__ int2 key_tiles(int qs, int N, int wl, int wr, int BN) {
  if (qs >= N) return make_int2(0, 0);
  const int2 kr = window_keys(qs, min(N, qs + 128), N, wl, wr);
  return make_int2(kr.x / BN, (kr.y + BN - 1) / BN);
}

// =====================================================================
// One query tile per CTA, double-buffered S (large head dimension).
// =====================================================================
template <typename T, int D, int BC, int NS>
struct SingleCfg {
  static constexpr bool FP8 = sizeof(T) == 1;  // e4m3 inputs, kind::f8f6f4 products
  static constexpr int ES = sizeof(T);
  static constexpr int ROWB = D * ES;
  static constexpr int NCHUNK = ROWB / 128;
  static constexpr int QCHUNK = 128 * 128;   // chunk of the 128-row Q tile
  static constexpr int KCHUNK = BC * 128;    // chunk of a BC-row K/V tile
  static constexpr int QTILE = 128 * ROWB;
  static constexpr int KTILE = BC * ROWB;
  static constexpr int QK_STEPS = ROWB / 32;
  static constexpr int PV_ROWS = 32 / ES;    // V rows consumed per P V step
  // e4m3: P is split into two e4m3 terms (high and residual), each multiplied by V
  static constexpr int PV_STEPS = (FP8 ? 2 : 1) * BC / PV_ROWS;
  static constexpr int EPC = 128 / ES;       // elements per 128-byte chunk
  static constexpr int S_COL = 0;            // S buffers at 0 and BC
  // D <= 128: S[2] | O in 256 columns, so that two CTAs share an SM's TMEM
  static constexpr int CTAS_PER_SM = D <= 128 ? 2 : 1;
  static constexpr int O_COL = D <= 128 ? 2 * BC : 256;
  static constexpr int TMEM_COLS = D <= 128 ? 256 : 512;
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_KV = QTILE;
  static constexpr int SMEM_BAR = SMEM_KV + NS * KTILE;
  // q_full, kv_full[NS], kv_empty[NS], s_full[2], p_full[2], o_full, done.
  // p_full alternates by key tile: S(j+1) is computed before P(j) is complete,
  // so a warp may arrive for tile j + 1 before the last warp arrives for j.
  // kv_empty of a V slot also tells the correction that P V of its tile is
  // complete.
  static constexpr int BAR_Q = 0;
  static constexpr int BAR_KVF = 1;
  static constexpr int BAR_KVE = 1 + NS;
  static constexpr int BAR_S = 1 + 2 * NS;
  static constexpr int BAR_P = 3 + 2 * NS;
  static constexpr int BAR_O = 5 + 2 * NS;
  static constexpr int BAR_DONE = 6 + 2 * NS;
  static constexpr int NBAR = 7 + 2 * NS;
  static constexpr int SMEM_MISC = SMEM_BAR + 8 * NBAR;
  static constexpr int SMEM_BITS = SMEM_MISC + 16;  // block-sparse: marked 128-key blocks
  static constexpr int SMEM_BYTES = SMEM_BITS + 4 * kMaskWords + 1024;
  static constexpr int THREADS = 256;
  static_assert(2 * BC <= O_COL && O_COL + D <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(sizeof(T) == 2 || (FP8 && D == 128), "bf16, or e4m3 at D = 128");
  // two co-resident CTAs: 228 KB of shared memory per SM, 1 KB reserved per CTA
  static_assert(CTAS_PER_SM == 1 || CTAS_PER_SM * (SMEM_BYTES + 1024) <= 233472,
                "two CTAs per SM");
};

// SPARSE: built for a block-sparse tile mask (p.bmask, 128 x 128 tile pairs):
// the BC-key tiles of unmarked 128-key blocks are skipped.
template <typename T, int D, int BC, int NS, bool SPARSE>
__global__ void __launch_bounds__(256, D <= 128 ? 2 : 1)
    fwd_single_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using C = SingleCfg<T, D, BC, NS>;
  static_assert(!SPARSE || 128 % BC == 0, "key tiles within 128-key mask blocks");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::SMEM_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::SMEM_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // head_major: grid (query blocks, Hq, B), the query tiles of one head are
  // dispatched together so its K and V stay in L2 while they are read
  // (DRAM reads of the 2x16x4096 causal forward 150 -> 101 MB).  Otherwise
  // grid (Hq, B, query blocks): the block index varies slowest so that every
  // head's longest causal CTAs are dispatched first (a head's longest tile
  // starting late leaves a tail that costs more than the re-reads save).
  const int qb = p.head_major ? gridDim.x - 1 - blockIdx.x : gridDim.z - 1 - blockIdx.z;
  const int h = p.head_major ? blockIdx.y : blockIdx.x;
  const int b = p.head_major ? blockIdx.z : blockIdx.y;
  const int hk = h / p.group;
  const int q0 = qb * 128;
  // key tiles [j0, j1) are visible to this query tile; the loops below run a
  // counter u over the computed ones (all of them without a block mask)
  const int2 ktr = key_tiles(q0, p.N, p.wl, p.wr, BC);
  const int j0 = ktr.x, j1 = ktr.y;
  constexpr int TPB = 128 / BC;  // key tiles per 128-key mask block
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + C::SMEM_BITS);
  if constexpr (SPARSE) {
    // bit kb: 128-key block kb is marked for this query tile (published to
    // every warp by the __syncthreads below)
    for (int wi = warp; wi < kMaskWords; wi += C::THREADS / 32) {
      const int kb = 32 * wi + lane;
      const bool on = kb < p.nt && qb < p.nt &&
                      p.bmask[((static_cast<long long>(b) * p.Hq + h) * p.nt + qb) * p.nt + kb] != 0;
      const uint32_t w = __ballot_sync(0xffffffffu, on);
      if (lane == 0) bits[wi] = w;
    }
  }
  // first computed key tile >= j (j1 if none)
  auto next_tile = [&](int j) -> int {
    j = max(j, j0);
    if constexpr (!SPARSE) {
      return min(j, j1);
    } else {
      if (j >= j1) return j1;
      // the first marked 128-key block at or after j's own
      const int kb = next_bit(bits, j / TPB, (j1 + TPB - 1) / TPB);
      return kb * TPB >= j1 ? j1 : max(j, kb * TPB);
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::BAR_Q), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(BAR(C::BAR_KVF + s), 1);
      mbar_init(BAR(C::BAR_KVE + s), 1);
    }
    mbar_init(BAR(C::BAR_S + 0), 1);
    mbar_init(BAR(C::BAR_S + 1), 1);
    mbar_init(BAR(C::BAR_P + 0), 4);
    mbar_init(BAR(C::BAR_P + 1), 4);
    mbar_init(BAR(C::BAR_O), 1);
    mbar_init(BAR(C::BAR_DONE), 1);
    *abort_flag = 0u;
    fence_barrier_init();
    fence_proxy_async_smem();
    // the Q tile's load starts before TMEM allocation and the block-wide sync;
    // Q is read once (L2 evict first), K and V by every query tile of the
    // head (evict last)
    mbar_expect_tx(BAR(C::BAR_Q), C::QTILE);
    tma_load_5d_hint(sbase + C::SMEM_Q, &tm_q, BAR(C::BAR_Q), 0, q0, 0, h, b,
                     l2_policy_evict_first());
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
  int n = 0;  // computed key tiles
  for (int j = next_tile(j0); j < j1; j = next_tile(j + 1)) ++n;

  if (warp < 4) {
    const int r = threadIdx.x & 127;
    const int qrow = q0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t o_addr = tmem + lane_base + C::O_COL;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int u = 0, j = next_tile(j0); u < n; ++u, j = next_tile(j + 1)) {
      const int buf = u & 1;
      const uint32_t s_addr = tmem + lane_base + C::S_COL + BC * buf;
      if (!W.wait_warp(BAR(C::BAR_S + buf), (u >> 1) & 1, 10)) { ok = false; break; }
      // S(u) is complete, so K_u's slot is free: released from here rather
      // than by a commit of its own (a commit costs the tensor pipe about as
      // much as a short product)
      if (threadIdx.x == 0) mbar_arrive(BAR(C::BAR_KVE + (2 * u) % NS));
      tc_fence_after();
      float s[BC];
      tmem_load_row<BC>(s_addr, s);
      apply_mask<BC>(s, col_window(BC * j, qrow, p.N, p.wl, p.wr));
      float alpha;
      const bool rescaled =
          online_softmax_step<BC, kSoftExp8, C::FP8 ? kP8Tau : static_cast<int>(kRescaleLog2)>(
              s, p.c, m, l, alpha);
      if constexpr (C::FP8) {
        tmem_store_p8<BC>(s_addr, s);
      } else {
        tmem_store_p<BC, false>(s_addr, s);
      }
      if (rescaled && u > 0) {
        // O must hold every P V product up to tile u-1 before it is rescaled.
        // V_{u-1}'s slot frees when P(u-1) V_{u-1} is complete (the same
        // event, one commit fewer per key tile than a barrier of its own:
        // measured 1-3 % faster); the slot's next release needs P of a later
        // tile, so its parity cannot alias
        const int it = 2 * (u - 1) + 1;
        if (!W.wait_warp(BAR(C::BAR_KVE + it % NS), static_cast<uint32_t>(it / NS) & 1u, 11)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_scale_row<D>(o_addr, alpha);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::BAR_P + (u & 1)));
    }
    if (ok && n == 0) {
      store_empty_row<__nv_bfloat16, D>(p, b, h, qrow);  // O is bf16 for either input
    } else if (ok && W.wait_warp(BAR(C::BAR_O), 0, 20)) {
      tc_fence_after();
      // O / l through TMA stores ({64, 32} boxes) staged in this warp's rows of
      // Q (every MMA reading Q is complete).  bf16: box k in Q's chunk k (one
      // chunk per 64 columns), so the boxes go out back to back; e4m3 (Q is
      // one chunk): every box in chunk 0, each waiting for the previous one
      static_assert(C::FP8 || C::NCHUNK == D / 64, "one Q chunk per output box");
      uint8_t* stage = smem + C::SMEM_Q + warp * 32 * 128;
      tmem_rows_tma_store<D>(o_addr, stage, &tm_o, 0, q0 + warp * 32, h, b,
                             l > 0.f ? p.o_mul / l : 0.f, C::FP8 ? 0u : C::QCHUNK);
      if (qrow < p.N)
        p.lse[(static_cast<long long>(b) * p.Hq + h) * p.N + qrow] =
            l > 0.f ? m * p.scale + logf(l) : -INFINITY;
      if (lane == 0) bulk_wait_read_all();  // the staging rows stay valid until read
      __syncwarp();
    }
  } else if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t pol_kv = l2_policy_evict_last();
      int it = 0;
      for (int u = 0, j = next_tile(j0); u < n && !W.aborted(); ++u, j = next_tile(j + 1)) {
        for (int kv = 0; kv < 2; ++kv, ++it) {
          const int slot = it % NS;
          const uint32_t ph = static_cast<uint32_t>(it / NS) & 1u;
          if (!W.wait(BAR(C::BAR_KVE + slot), ph ^ 1u, 30)) break;
          if ((p.debug_flags & 1) && kv == 1 && u == 0) continue;
          mbar_expect_tx(BAR(C::BAR_KVF + slot), C::KTILE);
          tma_load_5d_hint(sbase + C::SMEM_KV + slot * C::KTILE, kv ? &tm_v : &tm_k,
                           BAR(C::BAR_KVF + slot), 0, BC * j, 0, hk, b, pol_kv);
        }
      }
      const int issued = it;
      W.drain(BAR(C::BAR_Q), 0, 31);
      for (int s = 0; s < NS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / NS) * NS;
        W.drain(BAR(C::BAR_KVF + s), static_cast<uint32_t>(last / NS) & 1u, 32);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t fmt = C::FP8 ? 0u : 1u;  // e4m3 or bf16
      constexpr uint32_t idesc_s = idesc_make(128, BC, fmt, false, false);
      constexpr uint32_t idesc_o = idesc_make(128, D, fmt, false, true);
      auto kslot = [&](int j) { return (2 * j) % NS; };
      auto kph = [&](int j) { return static_cast<uint32_t>((2 * j) / NS) & 1u; };
      auto vslot = [&](int j) { return (2 * j + 1) % NS; };
      auto vph = [&](int j) { return static_cast<uint32_t>((2 * j + 1) / NS) & 1u; };
      const SDesc qa = sdesc_base(sbase + C::SMEM_Q, 16, 1024);
      auto issue_s = [&](int buf, int slot) {
        const SDesc kb = sdesc_base(sbase + C::SMEM_KV + slot * C::KTILE, 16, 1024);
        const uint32_t d = tmem + C::S_COL + BC * buf;
#pragma unroll
        for (int ks = 0; ks < C::QK_STEPS; ++ks) {
          const uint32_t qoff = (ks >> 2) * C::QCHUNK + (ks & 3) * 32;
          const uint32_t koff = (ks >> 2) * C::KCHUNK + (ks & 3) * 32;
          if constexpr (C::FP8) {
            mma_ss_f8(d, sdesc_at(qa, qoff), sdesc_at(kb, koff), idesc_s, ks > 0);
          } else {
            mma_ss<false>(d, sdesc_at(qa, qoff), sdesc_at(kb, koff), idesc_s, ks > 0);
          }
        }
      };
      auto issue_pv = [&](int buf, int slot, bool acc) {
        const SDesc vb = sdesc_base(sbase + C::SMEM_KV + slot * C::KTILE, C::KCHUNK, 1024);
        const uint32_t a = tmem + C::S_COL + BC * buf;
        const uint32_t acc0 = acc ? 1u : 0u;
#pragma unroll
        for (int ks = 0; ks < C::PV_STEPS; ++ks) {
          if constexpr (C::FP8) {
            // steps over P's high terms (TMEM columns [0, BC/4)), then its
            // residuals ([BC/4, BC/2)), both against the same V rows
            constexpr int VSTEPS = BC / C::PV_ROWS;
            mma_ts_f8(tmem + C::O_COL, a + 8u * ks,
                      sdesc_at(vb, (ks % VSTEPS) * C::PV_ROWS * 128), idesc_o, ks > 0 ? 1u : acc0);
          } else {
            mma_ts<false>(tmem + C::O_COL, a + 8u * ks, sdesc_at(vb, ks * C::PV_ROWS * 128),
                          idesc_o, ks > 0 ? 1u : acc0);
          }
        }
      };
      bool ok = n > 0 && W.wait(BAR(C::BAR_Q), 0, 40) &&
                W.wait(BAR(C::BAR_KVF + kslot(0)), kph(0), 41);
      if (ok) {
        tc_fence_after();
        issue_s(0, kslot(0));
        mma_commit(BAR(C::BAR_S + 0));  // also frees K_0's slot (softmax warp 0 arrives)
      }
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n) {
          if (!W.wait(BAR(C::BAR_KVF + kslot(j + 1)), kph(j + 1), 42)) { ok = false; break; }
          issue_s((j + 1) & 1, kslot(j + 1));
          mma_commit(BAR(C::BAR_S + ((j + 1) & 1)));
        }
        if (!W.wait(BAR(C::BAR_P + (j & 1)), (j >> 1) & 1, 43)) { ok = false; break; }
        if (!W.wait(BAR(C::BAR_KVF + vslot(j)), vph(j), 44)) { ok = false; break; }
        tc_fence_after();
        issue_pv(j & 1, vslot(j), j > 0);
        mma_commit(BAR(C::BAR_KVE + vslot(j)));
      }
      if (ok) mma_commit(BAR(C::BAR_O));
      mma_commit(BAR(C::BAR_DONE));
      W.drain(BAR(C::BAR_DONE), 0, 47);
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

}  // namespace eta
