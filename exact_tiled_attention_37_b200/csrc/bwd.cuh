// Backward attention kernels for sm_100a.
//
// Recompute-based backward from the saved per-row logsumexp: P is rebuilt
// tile by tile as exp2(S * scale * log2(e) - lse * log2(e)) and never stored.
// Five products per (key tile, query tile) pair as in the backward the
// FlashAttention (Metal Port) README describes for the official
// implementation (Documentation section: five GEMMs, scratch space for
// atomics and partial sums), with fp32 atomics for dQ:
//
//   S^T  = K Q_i^T            P^T  = exp2(S^T c - lse2_i)
//   dP^T = V dO_i^T           dS^T = P^T * (dP^T - Delta_i)
//   dV  += P^T dO_i           dK  += dS^T Q_i            (TMEM accumulators)
//   dQ_i^T = K^T dS^T   ->  atomically added (x scale) to an fp32 scratch dQ
//
// Kernels:
//  * bwd_preprocess_kernel: Delta = rowsum(dO * O) and lse2 = lse * log2(e)
//    per row (rows past N padded with Delta = 0, lse2 = +inf so that their P
//    is exactly 0), and zeroes the fp32 dQ scratch (head dimension 256).
//    D/8 threads per group of 4 rows.  Shared with the kernels of bwd_split.cuh.
//  * bwd_dkdv_kernel: one CTA per (batch, key/value head, 128-row key tile,
//    128-column slice of D); loops over the query heads of the GQA group and
//    the 64-row query tiles (causal: only tiles at or below the diagonal).
//    Roles: TMA producer warp, MMA warp, a 128-thread softmax warpgroup
//    (thread j owns key row j: computes P^T, dS^T rows into shared memory and
//    finally stores dK, dV), and a 128-thread dQ warpgroup (thread d owns
//    column d of dQ^T: drains dQ_i^T from TMEM and issues coalesced fp32
//    reductions into the scratch).
//    Shared memory holds one Q / dO tile, loaded in three parts: the D
//    chunks outside this CTA's slice are read only by S^T and dP^T, so the
//    next tile's part is loaded, and its S^T / dP^T steps run, under this
//    tile's softmax; the slice's own dO chunks follow once dV is done, its
//    Q chunks once dK is done.
//  * bwd_dq_finalize_kernel: dQ (bf16, caller's strides) from the scratch.
//
// TMEM (512 columns): ST[2] (64 each: S^T, then P^T and dS^T packed) |
// dPT[2] (64 each: dP^T, then dQ^T) | dV (128) | dK (128).
// Head dimension 256 is split into two 128-column slices (two CTAs per key
// tile, each recomputing S^T and dP^T over the full D): the TMEM-capacity
// analogue of the D-blocking the Metal port README describes.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "attn.h"
#include "ptx.cuh"

namespace eta {

#ifdef ETA_TRACE
// Debug builds only: per-role clock64() timelines of two CTAs of the dK/dV
// kernel ([cta][role][iteration][event]).
__device__ unsigned long long g_eta_trace[2][4][256][4];
#define ETA_TRACE_AT(cta, role, it, ev)                                          \
  do {                                                                          \
    if ((cta) >= 0 && (it) < 256) g_eta_trace[(cta)][(role)][(it)][(ev)] = clock64(); \
  } while (0)
#else
#define ETA_TRACE_AT(cta, role, it, ev) \
  do {                                  \
  } while (0)
#endif

// Rows of the per-row statistics are padded to a multiple of this.
constexpr int kBwdRowPad = 128;

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline size_t bwd_npad(int N) { return round_up(static_cast<size_t>(N), kBwdRowPad); }

// fp32 dQ scratch: only the fused kernel (head dimension 256) accumulates dQ
// there; for D <= 128 the row-parallel dQ kernel writes dQ directly.
inline size_t bwd_dqacc_bytes(int B, int Hq, int N, int D) {
  if (D <= 128) return 0;
  return round_up(static_cast<size_t>(B) * Hq * N * D * 4, 256);
}

inline size_t bwd_stat_bytes(int B, int Hq, int N) {
  return round_up(static_cast<size_t>(B) * Hq * bwd_npad(N) * 4, 256);
}

inline size_t bwd_workspace_bytes(int B, int Hq, int N, int D) {
  return bwd_dqacc_bytes(B, Hq, N, D) + 2 * bwd_stat_bytes(B, Hq, N);
}

struct BwdParams {
  const void* o;        // forward output [B, Hq, N, D]
  const void* dout;     // upstream gradient [B, Hq, N, D]
  const float* lse;     // [B, Hq, N]
  void* dq;             // [B, Hq, N, D] bf16
  void* dk;             // [B, Hkv, N, D] bf16
  void* dv;
  float* dqacc;         // [B, Hq, N, D] fp32 scratch
  float* delta;         // [B, Hq, Npad]
  float* lse2;          // [B, Hq, Npad]
  long long osb, osh, osn;
  long long dosb, dosh, dosn;
  long long dqsb, dqsh, dqsn;
  long long dksb, dksh, dksn;
  long long dvsb, dvsh, dvsn;
  int B, Hq, Hkv, N, D, Npad, group;
  int wl, wr;           // local window (query i sees keys [i - wl, i + wr]); -1 = unbounded
  float scale, c;       // c = scale * log2(e)
  int* status;
  unsigned long long wait_limit_ns;
  const uint8_t* bmask; // block-sparse tile mask [B, Hq, nt, nt] or null (D <= 128 only)
  int nt;               // ceil(N / 128)
  int debug_flags;      // bit 1: the dK/dV producer drops its second Q load (timeout test)
  int head_major;       // grid order of the dQ kernel (as FwdParams::head_major)
  // Stored dS^T tiles (head dimension 128, when the workspace holds them):
  // the dK/dV kernel writes each visible tile's dS^T (bf16, 32 KB) and the
  // dQ kernel sums dS K_j from them instead of recomputing S and dP.
  uint8_t* ds;          // null: the dQ kernel recomputes (seven products)
  long long ds_head;    // tiles per (batch, query head)
  int ds_tri;           // 1: causal triangle, slot i (i + 1) / 2 + j
  int ds_w;             // 0: band of ds_w slots per query tile, slot i ds_w + j - j_lo(i)
};

// ---------------------------------------------------------------- preprocess
// A group of D/8 threads covers kPrepRows consecutive rows, each thread
// reading 16 bytes of O and of dO per row; all of a thread's loads are issued
// before the first use, for enough bytes in flight to stream O and dO at HBM
// speed.  Rows past N get Delta = 0, lse2 = +inf.
constexpr int kPrepRows = 4;
static_assert(kBwdRowPad % kPrepRows == 0, "row groups never straddle a head");

template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const BwdParams p) {
  constexpr int TPR = D / 8;  // threads per row (8, 16 or 32)
  constexpr int R = kPrepRows;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row0 = t / TPR * R;  // first of R rows over B * Hq * Npad
  const int part = static_cast<int>(t % TPR);
  const long long rows = static_cast<long long>(p.B) * p.Hq * p.Npad;
  // (Npad is a multiple of R, so the R rows share one (batch, head); the
  // guard keeps every lane in the shuffles below)
  const bool in_range = row0 < rows;
  const int bh = static_cast<int>(row0 / p.Npad);
  const int i0 = static_cast<int>(row0 % p.Npad);
  const int b = bh / p.Hq, h = bh % p.Hq;
  const __nv_bfloat16* orow = static_cast<const __nv_bfloat16*>(p.o) + b * p.osb + h * p.osh +
                              static_cast<long long>(i0) * p.osn + 8 * part;
  const __nv_bfloat16* drow = static_cast<const __nv_bfloat16*>(p.dout) + b * p.dosb +
                              h * p.dosh + static_cast<long long>(i0) * p.dosn + 8 * part;
  uint4 ov[R], dv[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const bool live = in_range && i0 + r < p.N;
    ov[r] = live ? *reinterpret_cast<const uint4*>(orow + r * p.osn) : make_uint4(0, 0, 0, 0);
    dv[r] = live ? *reinterpret_cast<const uint4*>(drow + r * p.dosn) : make_uint4(0, 0, 0, 0);
  }
  // zero this part of the fp32 dQ scratch rows (when dQ is accumulated there)
  if (p.dqacc) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (in_range && i0 + r < p.N) {
        float4* z = reinterpret_cast<float4*>(
            p.dqacc + (static_cast<long long>(bh) * p.N + i0 + r) * D + 8 * part);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov[r]);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv[r]);
    acc[r] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 of = __bfloat1622float2(o2[e]);
      const float2 df = __bfloat1622float2(d2[e]);
      acc[r] = fmaf(of.x, df.x, acc[r]);
      acc[r] = fmaf(of.y, df.y, acc[r]);
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1)
      acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], off);
  }
  // thread r of the group writes row r
  if (in_range && part < R) {
    float a = acc[0];
#pragma unroll
    for (int r = 1; r < R; ++r)
      if (part == r) a = acc[r];
    const int i = i0 + part;
    p.delta[row0 + part] = a;
    // rows past N, and rows that saw no key (lse = -inf), get lse2 = +inf so
    // that their P is exactly 0
    const float l = i < p.N ? p.lse[static_cast<long long>(bh) * p.N + i] : -INFINITY;
    p.lse2[row0 + part] = l > -INFINITY ? l * 1.4426950408889634f : INFINITY;
  }
}

// ---------------------------------------------------------------- dQ finalize
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_finalize_kernel(const BwdParams p) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  constexpr int VEC = 8;
  const long long per_row = D / VEC;
  const long long total = static_cast<long long>(p.B) * p.Hq * p.N * per_row;
  if (idx >= total) return;
  const long long row = idx / per_row;
  const int col = static_cast<int>(idx % per_row) * VEC;
  const int i = static_cast<int>(row % p.N);
  const int bh = static_cast<int>(row / p.N);
  const int b = bh / p.Hq, h = bh % p.Hq;
  const float4* src = reinterpret_cast<const float4*>(p.dqacc + row * D + col);
  const float4 a = src[0], c = src[1];
  uint4 w;
  w.x = pack_bf16x2(a.x, a.y);
  w.y = pack_bf16x2(a.z, a.w);
  w.z = pack_bf16x2(c.x, c.y);
  w.w = pack_bf16x2(c.z, c.w);
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.dq) + b * p.dqsb + h * p.dqsh + i * p.dqsn + col;
  *reinterpret_cast<uint4*>(dst) = w;
}

// ---------------------------------------------------------------- dK / dV (+ dQ reductions)
template <int DFULL, int NQS, int NPB>
struct BwdCfg {
  static constexpr int BC = 128;                 // key rows per CTA
  static constexpr int BR = 64;                  // query rows per iteration
  static constexpr int DH = 128;                 // D slice of dK/dV/dQ per CTA
  static constexpr int DSPLIT = DFULL / DH;
  static constexpr int ROWB = DFULL * 2;
  static constexpr int NCHUNK = ROWB / 128;
  static constexpr int KCHUNK = BC * 128;        // 16 KB
  static constexpr int QCHUNK = BR * 128;        // 8 KB
  static constexpr int KTILE = BC * ROWB;
  static constexpr int QTILE = BR * ROWB;
  static constexpr int PTILE = BC * BR * 2;      // 16 KB dS^T: one 128-byte row per key row
  static constexpr int KSTEPS = ROWB / 32;       // S^T / dP^T MMAs over D
  // dQ_i partials: each drain warp stages its 32 columns x 64 rows (8 KB) in
  // shared memory and hands them to the TMA engine as one tiled bulk
  // reduction (when shared memory allows: D = 128), otherwise fp32
  // reductions from registers.
  static constexpr bool DQ_BULK = DFULL == DH;
  static constexpr int DQWARP = BR * 32 * 4;                 // 8 KB per drain warp
  static constexpr int DQTILE = DQ_BULK ? 4 * DQWARP : 0;    // 32 KB
  // TMEM columns
  static constexpr int T_ST = 0, T_DPT = 128, T_DV = 256, T_DK = 384, TMEM_COLS = 512;
  // shared memory
  static constexpr int S_K = 0;
  static constexpr int S_V = S_K + KTILE;
  static constexpr int S_Q = S_V + KTILE;                  // [NQS] Q tiles
  static constexpr int S_DO = S_Q + NQS * QTILE;           // [NQS] dO tiles
  static constexpr int S_DS = S_DO + NQS * QTILE;          // [NPB] dS^T
  static constexpr int S_DQ = S_DS + NPB * PTILE;          // dQ staging
  static constexpr int S_STAT = S_DQ + DQTILE;             // [NQS] lse2[64], delta[64]
  static constexpr int S_BAR = S_STAT + NQS * 512;
  static constexpr int B_KV = 0;
  static constexpr int B_QF = 1;
  static constexpr int B_QE = 1 + NQS;
  static constexpr int B_SP = 1 + 2 * NQS;                // [2]
  static constexpr int B_DS = 3 + 2 * NQS;                // [NPB]
  static constexpr int B_PE = 3 + 2 * NQS + NPB;          // [NPB]
  static constexpr int B_DQF = 3 + 2 * NQS + 2 * NPB;     // [2]
  static constexpr int B_DQE = 5 + 2 * NQS + 2 * NPB;     // [2]
  static constexpr int B_KVD = 7 + 2 * NQS + 2 * NPB;     // dK/dV accumulated
  static constexpr int B_DONE = 8 + 2 * NQS + 2 * NPB;
  // the Q / dO chunks outside this CTA's D slice (read only by S^T and dP^T)
  // have barriers of their own: they are free again as soon as those two
  // products are done, while the slice's own chunks wait for dV and dK
  // B_WF / B_WE: the slice's own Q chunks and the row statistics (free
  // after dK); B_QF / B_QE: the slice's own dO chunks (free after dV)
  static constexpr int B_OF = 9 + 2 * NQS + 2 * NPB;
  static constexpr int B_OE = 10 + 2 * NQS + 2 * NPB;
  static constexpr int B_WF = 11 + 2 * NQS + 2 * NPB;
  static constexpr int B_WE = 12 + 2 * NQS + 2 * NPB;
  // B_SP[2] signals S^T complete, B_SPD[2] dP^T complete
  static constexpr int B_SPD = 13 + 2 * NQS + 2 * NPB;   // [2]
  static constexpr int NBAR = 15 + 2 * NQS + 2 * NPB;
  static constexpr int S_MISC = S_BAR + 8 * NBAR;
  static constexpr int SMEM_BYTES = S_MISC + 16 + 1024;
  // warps: 0-3 softmax (query columns 0-31 of every tile), 4-7 dQ drain,
  // 8-11 softmax (columns 32-63), 12 TMA producer, 13 MMA issuer / TMEM
  // owner, 14-15 idle
  static constexpr int THREADS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// P^T for 32 query columns [c0, c0 + 32) of this thread's key row: loads S^T
// from TMEM and applies exp2(S^T c - lse2) and the window mask, into pv.
__device__ __forceinline__ void bwd_row_p(uint32_t st_addr, int c0, const float* lse2, float c,
                                          int ilo, int ihi, float (&pv)[32]) {
  uint32_t rs[32];
  tmem_ld32(st_addr + c0, rs);
  tmem_wait_ld();
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float2 l2 = *reinterpret_cast<const float2*>(lse2 + c0 + i);
    const float2 x = ffma2(make_float2(u2f(rs[i]), u2f(rs[i + 1])), c2, make_float2(-l2.x, -l2.y));
    pv[i] = (c0 + i < ilo || c0 + i > ihi) ? 0.f : ex2(x.x);
    pv[i + 1] = (c0 + i + 1 < ilo || c0 + i + 1 > ihi) ? 0.f : ex2(x.y);
  }
}

// dS^T = P^T * (dP^T - Delta) for the same columns: loads dP^T from TMEM and
// writes P^T and dS^T as bf16 pairs into the 32 S^T columns read before (P^T
// at columns c0 .. c0 + 15, dS^T at c0 + 16 .. c0 + 31: the A operands of
// dV += P^T dO and dK += dS^T Q), and dS^T also as a bf16 shared-memory row
// (4 swizzled 16-byte chunks: the B operand of dQ^T = K^T dS^T).  The dP^T
// columns are left free for dQ^T.
__device__ __forceinline__ void bwd_row_ds(uint32_t st_addr, uint32_t dpt_addr, int c0,
                                           const float* dlt, const float (&pv)[32], uint8_t* drow,
                                           int swz) {
  uint32_t rd[32];
  tmem_ld32(dpt_addr + c0, rd);
  tmem_wait_ld();
  uint32_t pk[16], dk[16];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t dw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = 8 * u + 2 * e;  // column within this half
      const float2 dd = *reinterpret_cast<const float2*>(dlt + c0 + i);
      const float2 g = fsub2(make_float2(u2f(rd[i]), u2f(rd[i + 1])), dd);
      pk[4 * u + e] = pack_bf16x2(pv[i], pv[i + 1]);
      dw[e] = pack_bf16x2(pv[i] * g.x, pv[i + 1] * g.y);
      dk[4 * u + e] = dw[e];
    }
    const int chunk = (c0 >> 3) + u;  // 16-byte chunk index within the 128-byte row
    const int off = (chunk ^ swz) * 16;
    *reinterpret_cast<uint4*>(drow + off) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
  }
  tmem_st16(st_addr + c0, pk);
  tmem_st16(st_addr + c0 + 16, dk);
}

template <int DFULL, int NQS, int NPB>
__global__ void __launch_bounds__(512, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using C = BwdCfg<DFULL, NQS, NPB>;
  static_assert(NQS == 1 && C::DSPLIT == 2, "one Q/dO stage, split into the two D slices");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::S_BAR;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::S_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::S_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (Hkv * D-slices, B, key tiles).  Masked problems: the key tile
  // varies slowest, so causal tile 0 (the most work) of every head is
  // dispatched first.  Unmasked problems (equal work per CTA): the key tile
  // varies fastest, so the CTAs of one head run together and share its Q /
  // dO tiles and dQ rows in L2.
  const bool kt_fast = p.wl < 0 && p.wr < 0;
  const int lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  const int kt = kt_fast ? lin % gridDim.z : blockIdx.z;
  const int hk = kt_fast ? lin / gridDim.z / C::DSPLIT % p.Hkv : blockIdx.x / C::DSPLIT;
  const int half = kt_fast ? lin / gridDim.z % C::DSPLIT : blockIdx.x % C::DSPLIT;
  const int b = kt_fast ? lin / gridDim.z / C::DSPLIT / p.Hkv : blockIdx.y;
  const int k0 = kt * C::BC;
  // queries that see any key of [k0, k0 + BC): key j is visible to query i iff
  // j - wr <= i <= j + wl
  const int q_lo = p.wr < 0 ? 0 : max(0, k0 - p.wr);
  const int q_hi = p.wl < 0 ? p.N : min(p.N, min(p.N, k0 + C::BC) + p.wl);
  const int i_first = q_lo / C::BR;
  const int per_head = (q_hi + C::BR - 1) / C::BR - i_first;
  const int n = per_head * p.group;  // iterations: query heads of the group x query tiles

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_KV), 1);
    for (int s = 0; s < NQS; ++s) {
      mbar_init(BAR(C::B_QF + s), 1);
      mbar_init(BAR(C::B_QE + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(C::B_SP + s), 1);
      mbar_init(BAR(C::B_SPD + s), 1);
      mbar_init(BAR(C::B_DQF + s), 1);
      mbar_init(BAR(C::B_DQE + s), 4);
    }
    for (int s = 0; s < NPB; ++s) {
      mbar_init(BAR(C::B_DS + s), 8);
      mbar_init(BAR(C::B_PE + s), 1);
    }
    mbar_init(BAR(C::B_KVD), 1);
    mbar_init(BAR(C::B_DONE), 1);
    mbar_init(BAR(C::B_OF), 1);
    mbar_init(BAR(C::B_OE), 1);
    mbar_init(BAR(C::B_WF), 1);
    mbar_init(BAR(C::B_WE), 1);
    *abort_flag = 0u;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, p.status, p.wait_limit_ns};

#ifdef ETA_TRACE
  const int tcta = lin == 0 ? 0 : (lin == 37 ? 1 : -1);
#else
  const int tcta = -1;
#endif
  (void)tcta;
  // iteration -> (query head, query tile)
  auto head_of = [&](int it) { return hk * p.group + it / per_head; };
  auto qtile_of = [&](int it) { return i_first + it % per_head; };

  if (warp < 4 || (warp >= 8 && warp < 12)) {
    // ------------------------------------------------ P^T / dS^T rows, then dK / dV epilogue
    const int par = warp < 4 ? 0 : 1;   // this warpgroup's half of the 64 query columns
    const int j = threadIdx.x & 127;    // key row within the tile == TMEM lane
    const int jg = k0 + j;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int buf = it & 1, stage = it % NQS, pb = it % NPB;
      // S^T complete, and the row statistics (loaded with the slice's Q chunks)
      if (!W.wait_warp(BAR(C::B_SP + buf), (it >> 1) & 1, 60)) { ok = false; break; }
      if (!W.wait_warp(BAR(C::B_WF), it & 1, 61)) { ok = false; break; }
      if ((threadIdx.x & 127) == 0) ETA_TRACE_AT(tcta, 0, it, 0);
      tc_fence_after();
      const float* lse2 = reinterpret_cast<const float*>(smem + C::S_STAT + stage * 512);
      const float* dlt = lse2 + 64;
      const int ig0 = qtile_of(it) * C::BR;
      // window: query ig0 + i sees key jg iff jg - wr <= ig0 + i <= jg + wl
      const int ilo = p.wr < 0 ? -(1 << 30) : jg - p.wr - ig0;
      const int ihi = p.wl < 0 ? (1 << 30) : jg + p.wl - ig0;
      uint8_t* drow = smem + C::S_DS + pb * C::PTILE + j * 128;
      const uint32_t st_addr = tmem + lane_base + C::T_ST + 64 * buf;
      const uint32_t dpt_addr = tmem + lane_base + C::T_DPT + 64 * buf;
      float pv[32];
      bwd_row_p(st_addr, 32 * par, lse2, p.c, ilo, ihi, pv);
      // dP^T complete, and the MMAs that read this dS^T buffer NPB iterations
      // ago done
      if (!W.wait_warp(BAR(C::B_SPD + buf), (it >> 1) & 1, 64)) { ok = false; break; }
      if (!W.wait_warp(BAR(C::B_PE + pb), ((it / NPB) & 1) ^ 1, 62)) { ok = false; break; }
      if ((threadIdx.x & 127) == 0) ETA_TRACE_AT(tcta, 0, it, 1);
      tc_fence_after();
      bwd_row_ds(st_addr, dpt_addr, 32 * par, dlt, pv, drow, j & 7);
      if ((threadIdx.x & 127) == 0) ETA_TRACE_AT(tcta, 0, it, 2);
      tmem_wait_st();
      fence_proxy_async_smem();  // generic-proxy smem writes -> tensor core reads
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_DS + pb));
      if ((threadIdx.x & 127) == 0) ETA_TRACE_AT(tcta, 0, it, 3);
    }
    if (ok && W.wait_warp(BAR(C::B_KVD), 0, 63)) {
      tc_fence_after();
      // even warpgroup stores dV, odd warpgroup stores dK (x scale)
      const bool valid = jg < p.N;
      __nv_bfloat16* row =
          par == 0 ? static_cast<__nv_bfloat16*>(p.dv) + b * p.dvsb + hk * p.dvsh +
                         static_cast<long long>(jg) * p.dvsn + half * C::DH
                   : static_cast<__nv_bfloat16*>(p.dk) + b * p.dksb + hk * p.dksh +
                         static_cast<long long>(jg) * p.dksn + half * C::DH;
      const float mul = par ? p.scale : 1.f;
      const uint32_t col = par ? C::T_DK : C::T_DV;
#pragma unroll 1
      for (int c = 0; c < C::DH / 32; ++c) {
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
    }
  } else if (warp < 8) {
    // ------------------------------------------------ dQ^T drain -> fp32 reductions
    const int dd = threadIdx.x - 128;  // column of this CTA's D slice == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int dw = warp & 3;  // drain warp: columns [32 dw, 32 dw + 32) of the D slice
    float* stage_dq = reinterpret_cast<float*>(smem + C::S_DQ + dw * C::DQWARP);
    for (int it = 0; it < n; ++it) {
      const int buf = it & 1;
      if (!W.wait_warp(BAR(C::B_DQF + buf), (it >> 1) & 1, 70)) break;
      if (threadIdx.x == 128) ETA_TRACE_AT(tcta, 1, it, 0);
      tc_fence_after();
      float v[64];
      tmem_load_row<64>(tmem + lane_base + C::T_DPT + 64 * buf, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::B_DQE + buf));
      if (threadIdx.x == 128) ETA_TRACE_AT(tcta, 1, it, 1);
      const int h = head_of(it);
      const int ig0 = qtile_of(it) * C::BR;
      const int imax = min(64, p.N - ig0);
      float* dst = p.dqacc + (static_cast<long long>(b * p.Hq + h) * p.N + ig0) * DFULL;
      if constexpr (C::DQ_BULK) {
        // this warp's previous reduction must have finished reading its staging box
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 64; ++i) stage_dq[i * 32 + lane] = v[i] * p.scale;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // box of 32 columns x 64 rows of the (D, N, B*Hq) scratch; rows past N are skipped
          tma_reduce_add_3d(&tm_dq, smem_u32(stage_dq), half * C::DH + 32 * dw, ig0, b * p.Hq + h);
          bulk_commit();
        }
        (void)imax;
        (void)dst;
      } else {
        float* col = dst + half * C::DH + dd;
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i < imax) atomicAdd(col + static_cast<long long>(i) * DFULL, v[i] * p.scale);
      }
      if (threadIdx.x == 128) ETA_TRACE_AT(tcta, 1, it, 2);
    }
    if constexpr (C::DQ_BULK) {
      if (lane == 0) bulk_wait_all();
      __syncwarp();
    }
  } else if (warp == 12) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_expect_tx(BAR(C::B_KV), 2 * C::KTILE);
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d(sbase + C::S_K + c * C::KCHUNK, &tm_k, BAR(C::B_KV), c * 64, k0, hk, b);
        tma_load_4d(sbase + C::S_V + c * C::KCHUNK, &tm_v, BAR(C::B_KV), c * 64, k0, hk, b);
      }
      // Q / dO chunks 2 half, 2 half + 1 are this CTA's D slice ("own"), the
      // other two are read only by S^T and dP^T
      const int c_own = 2 * half, c_oth = 2 - 2 * half;
      int it = 0, oth_issued = 0, q_issued = 0;
      for (; it < n; ++it) {
        const int h = head_of(it);
        const int ig0 = qtile_of(it) * C::BR;
        if (!W.wait(BAR(C::B_OE), (it & 1) ^ 1, 80)) break;
        ETA_TRACE_AT(tcta, 3, it, 0);
        mbar_expect_tx(BAR(C::B_OF), 4 * C::QCHUNK);
        for (int c = c_oth; c < c_oth + 2; ++c) {
          tma_load_4d(sbase + C::S_Q + c * C::QCHUNK, &tm_q, BAR(C::B_OF), c * 64, ig0, h, b);
          tma_load_4d(sbase + C::S_DO + c * C::QCHUNK, &tm_do, BAR(C::B_OF), c * 64, ig0, h, b);
        }
        ++oth_issued;
        if (!W.wait(BAR(C::B_WE), (it & 1) ^ 1, 84)) break;
        ETA_TRACE_AT(tcta, 3, it, 1);
        mbar_expect_tx(BAR(C::B_WF), 2 * C::QCHUNK + 512);
        for (int c = c_own; c < c_own + 2; ++c)
          if (!((p.debug_flags & 2) && it == 1))
            tma_load_4d(sbase + C::S_Q + c * C::QCHUNK, &tm_q, BAR(C::B_WF), c * 64, ig0, h, b);
        const long long srow = static_cast<long long>(b * p.Hq + h) * p.Npad + ig0;
        bulk_load(sbase + C::S_STAT, p.lse2 + srow, 256, BAR(C::B_WF));
        bulk_load(sbase + C::S_STAT + 256, p.delta + srow, 256, BAR(C::B_WF));
        ++q_issued;
        if (!W.wait(BAR(C::B_QE), (it & 1) ^ 1, 85)) break;
        ETA_TRACE_AT(tcta, 3, it, 2);
        mbar_expect_tx(BAR(C::B_QF), 2 * C::QCHUNK);
        for (int c = c_own; c < c_own + 2; ++c)
          tma_load_4d(sbase + C::S_DO + c * C::QCHUNK, &tm_do, BAR(C::B_QF), c * 64, ig0, h, b);
      }
      W.drain(BAR(C::B_KV), 0, 81);
      if (q_issued > 0) W.drain(BAR(C::B_WF), static_cast<uint32_t>(q_issued - 1) & 1u, 82);
      if (it > 0) W.drain(BAR(C::B_QF), static_cast<uint32_t>(it - 1) & 1u, 86);
      if (oth_issued > 0) W.drain(BAR(C::B_OF), static_cast<uint32_t>(oth_issued - 1) & 1u, 83);
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_make(128, 64, 1u, false, false);      // S^T, dP^T
      constexpr uint32_t id_kv = idesc_make(128, C::DH, 1u, false, true);   // dV, dK
      constexpr uint32_t id_q = idesc_make(128, 64, 1u, true, true);        // dQ^T
      const SDesc dK = sdesc_base(sbase + C::S_K, 16, 1024);
      const SDesc dV = sdesc_base(sbase + C::S_V, 16, 1024);
      // K^T for dQ^T: MN-major view of this CTA's D slice of the K tile
      const SDesc dKt = sdesc_base(sbase + C::S_K + half * 2 * C::KCHUNK, C::KCHUNK, 1024);
      // S^T (K Q_i^T) or dP^T (V dO_i^T) over the 64-column chunks c0, c0 + 1
      // of D (8 steps)
      auto issue_half = [&](bool dp, int it, int c0, bool first) {
        const SDesc a = dp ? dV : dK;
        const SDesc bq = sdesc_base(sbase + (dp ? C::S_DO : C::S_Q), 16, 1024);
        const uint32_t d = tmem + (dp ? C::T_DPT : C::T_ST) + 64 * (it & 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ko = (c0 + (kk >> 2)) * C::KCHUNK + (kk & 3) * 32;
          const uint32_t qo = (c0 + (kk >> 2)) * C::QCHUNK + (kk & 3) * 32;
          mma_ss<false>(d, sdesc_at(a, ko), sdesc_at(bq, qo), id_s, !first || kk > 0);
        }
      };
      const int c_own = 2 * half, c_oth = 2 - 2 * half;
      auto issue_other = [&](int it) {
        tc_fence_after();
        issue_half(false, it, c_oth, true);
        issue_half(true, it, c_oth, true);
        mma_commit(BAR(C::B_OE));
      };
      // this slice's chunks: S^T as soon as Q has arrived (the softmax starts
      // on P while dP^T runs), then dP^T
      auto issue_own = [&](int it) -> bool {
        if (!W.wait(BAR(C::B_WF), it & 1, 97)) return false;
        tc_fence_after();
        issue_half(false, it, c_own, false);
        mma_commit(BAR(C::B_SP + (it & 1)));
        if (!W.wait(BAR(C::B_QF), it & 1, 98)) return false;
        tc_fence_after();
        issue_half(true, it, c_own, false);
        mma_commit(BAR(C::B_SPD + (it & 1)));
        return true;
      };
      bool ok = W.wait(BAR(C::B_KV), 0, 90) && (n == 0 || W.wait(BAR(C::B_OF), 0, 91));
      if (ok && n > 0) {
        issue_other(0);
        ok = issue_own(0);
      }
      for (int it = 0; ok && it < n; ++it) {
        const int buf = it & 1, b1 = (it + 1) & 1, pb = it % NPB;
        ETA_TRACE_AT(tcta, 2, it, 0);
        // The next tile's S^T / dP^T over the other slice's chunks go into the
        // other TMEM buffers (once the dQ warpgroup has drained the dQ^T that
        // last used that dP^T buffer) and run under this tile's softmax, if
        // their chunks have landed; otherwise after this tile's products.
        bool other_issued = false;
        if (it + 1 < n && (it == 0 || mbar_test(BAR(C::B_DQE + b1), ((it - 1) >> 1) & 1)) &&
            mbar_test(BAR(C::B_OF), (it + 1) & 1)) {
          issue_other(it + 1);
          other_issued = true;
        }
        ETA_TRACE_AT(tcta, 2, it, 1);
        if (!W.wait(BAR(C::B_DS + pb), (it / NPB) & 1, 94)) { ok = false; break; }
        ETA_TRACE_AT(tcta, 2, it, 2);
        tc_fence_after();
        const SDesc dq = sdesc_base(sbase + C::S_Q + half * 2 * C::QCHUNK, C::QCHUNK, 1024);
        const SDesc ddo = sdesc_base(sbase + C::S_DO + half * 2 * C::QCHUNK, C::QCHUNK, 1024);
        const SDesc dds = sdesc_base(sbase + C::S_DS + pb * C::PTILE, C::PTILE, 1024);
        const uint32_t tst = tmem + C::T_ST + 64 * buf, tdp = tmem + C::T_DPT + 64 * buf;
        const uint32_t acc0 = it > 0 ? 1u : 0u;
        // P^T / dS^T of query rows [16 ks, 16 ks + 16) sit at S^T column
        // 32 (ks / 2) + 8 (ks % 2) (+ 16 for dS^T)
        // dK += dS^T Q_i with dS^T read from TMEM (K = 64 query rows, 4 steps of
        // 16); then the slice's Q chunks and the statistics are free
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ts<false>(tmem + C::T_DK, tst + 32 * (ks >> 1) + 16 + 8 * (ks & 1),
                        sdesc_at(dq, ks * 2048), id_kv, ks > 0 ? 1u : acc0);
        mma_commit(BAR(C::B_WE));
        // dV += P^T dO_i with P^T read from TMEM; then the slice's dO chunks are free
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ts<false>(tmem + C::T_DV, tst + 32 * (ks >> 1) + 8 * (ks & 1), sdesc_at(ddo, ks * 2048),
                        id_kv, ks > 0 ? 1u : acc0);
        mma_commit(BAR(C::B_QE));
        // dQ_i^T = K^T dS^T (K = 128 key rows, 8 steps of 16) into the consumed dP^T buffer
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss<false>(tdp, sdesc_at(dKt, ks * 2048), sdesc_at(dds, ks * 2048), id_q, ks > 0);
        mma_commit(BAR(C::B_DQF + buf));
        mma_commit(BAR(C::B_PE + pb));
        ETA_TRACE_AT(tcta, 2, it, 3);
        if (it + 1 < n) {
          if (!other_issued) {
            if (it >= 1 && !W.wait(BAR(C::B_DQE + b1), ((it - 1) >> 1) & 1, 92)) { ok = false; break; }
            if (!W.wait(BAR(C::B_OF), (it + 1) & 1, 93)) { ok = false; break; }
            issue_other(it + 1);
          }
          if (!issue_own(it + 1)) { ok = false; break; }
        }
      }
      if (ok) mma_commit(BAR(C::B_KVD));
      mma_commit(BAR(C::B_DONE));
      W.drain(BAR(C::B_DONE), 0, 95);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace eta
