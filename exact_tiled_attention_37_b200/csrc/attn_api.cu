// C ABI of the exact tiled attention library: argument validation, TMA
// tensor-map construction, tile-configuration choice by head dimension (the
// role the "parameter file" keyed by D plays in the FlashAttention (Metal
// Port) README, Documentation section, here a compile-time table) and kernel
// launches.  The library allocates no device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "bwd.cuh"
#include "bwd_split.cuh"
#include "bwd_kv3.cuh"
#include "bwd_dqs.cuh"
#include "fwd.cuh"
#include "fwd_pair.cuh"
#include "decode.cuh"
#include "fwd_fp32.cuh"

// Head dimension 128 backward: 1 = the dK/dV kernel with three Q stages
// (bwd_kv3.cuh), 0 = the two-stage one (bwd_split.cuh), kept for comparison.
#ifndef ETA_KV3
#define ETA_KV3 1
#endif

// Device status word: [0] code, [1] wait site, [2..3] block of the first failure.
__device__ int g_attn_status[4];

namespace {

__global__ void debug_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int n,
                                  int mode) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
  float2 r;
  if (mode == 1) {
    r = eta::exp2_poly2(make_float2(a, b));
  } else {
    r.x = eta::ex2(a);
    r.y = eta::ex2(b);
  }
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}

constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;  // 2 s
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};
std::atomic<int> g_debug_flags{0};
// Forward kernel for bf16, D = 128 without a block mask: 0 = the default, 1 =
// the single-CTA kernel, 2 = the CTA-pair kernel (selectable for comparisons).
std::atomic<int> g_fwd_variant{0};
std::atomic<void*> g_bwd_ev_start{nullptr};
std::atomic<void*> g_bwd_ev_stop{nullptr};
std::atomic<void*> g_bwd_q_ev_start{nullptr};
std::atomic<void*> g_bwd_q_ev_stop{nullptr};

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
std::mutex g_mu;

attn_status_t status_ptr(int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_status) != cudaSuccess) return ATTN_ERR_CUDA;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_status_ptr[dev];
  return ATTN_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks one [B, H, N, D] tensor: non-null, 16-byte aligned base, strides that
// are positive (where the dimension has more than one entry) multiples of 16
// bytes.
attn_status_t check_tensor(const attn_tensor_t& t, int B, int H, int N, int es) {
  if (!t.ptr) return ATTN_ERR_INVALID_ARG;
  if ((B > 1 && t.sb <= 0) || (H > 1 && t.sh <= 0) || (N > 1 && t.sn <= 0))
    return ATTN_ERR_INVALID_ARG;
  if (t.sb < 0 || t.sh < 0 || t.sn < 0) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(t.ptr)) return ATTN_ERR_MISALIGNED;
  if ((t.sb * es) % 16 || (t.sh * es) % 16 || (t.sn * es) % 16) return ATTN_ERR_MISALIGNED;
  return ATTN_OK;
}

// An output tensor must not overlap itself: otherwise two CTAs write the same
// elements and the result depends on their order.  Sufficient condition: with
// the dimensions of extent > 1 sorted by stride (D has stride 1), every stride
// reaches past the whole span of the dimensions inside it.
attn_status_t check_output_layout(const attn_tensor_t& t, int B, int H, int N, int D) {
  struct Dim { long long extent, stride; } d[4] = {{D, 1}, {N, t.sn}, {H, t.sh}, {B, t.sb}};
  Dim v[4];
  int n = 0;
  for (const Dim& x : d)
    if (x.extent > 1) v[n++] = x;
  std::sort(v, v + n, [](const Dim& a, const Dim& b) { return a.stride < b.stride; });
  long long span = 0;  // largest element offset reachable through the inner dimensions
  for (int i = 0; i < n; ++i) {
    if (v[i].stride <= span) return ATTN_ERR_INVALID_ARG;
    span += (v[i].extent - 1) * v[i].stride;
  }
  return ATTN_OK;
}

// 4-D TMA map over [B, H, N, D] (innermost first: D, N, H, B), 128-byte
// swizzle, boxes of (128 bytes of D) x box_rows rows.
attn_status_t make_map(CUtensorMap* m, const attn_tensor_t& t, int B, int H, int N, int D, int es,
                       int box_rows) {
  auto enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;
  int64_t sn = N > 1 ? t.sn : D;
  int64_t sh = H > 1 ? t.sh : sn * N;
  int64_t sb = B > 1 ? t.sb : sh * H;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(sn * es), static_cast<cuuint64_t>(sh * es),
                           static_cast<cuuint64_t>(sb * es)};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / es), static_cast<cuuint32_t>(box_rows), 1u, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUtensorMapDataType dt = es == 2   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUresult r = enc(m, dt,
                   4, t.ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 5-D TMA map over [B, H, N, D] seen as (128-byte chunk of a row, row, chunk,
// head, batch): one box of box_rows rows x box_chunks chunks is a whole tile
// in the chunked shared-memory layout [chunk][row][128 bytes].
attn_status_t make_tile_map(CUtensorMap* m, const attn_tensor_t& t, int B, int H, int N, int D,
                            int es, int box_rows, int box_chunks) {
  auto enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;
  int64_t sn = N > 1 ? t.sn : D;
  int64_t sh = H > 1 ? t.sh : sn * N;
  int64_t sb = B > 1 ? t.sb : sh * H;
  const int epc = 128 / es;  // elements per chunk
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(epc), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(D / epc), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(sn * es), 128u,
                           static_cast<cuuint64_t>(sh * es), static_cast<cuuint64_t>(sb * es)};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(epc), static_cast<cuuint32_t>(box_rows),
                       static_cast<cuuint32_t>(box_chunks), 1u, 1u};
  cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  const CUtensorMapDataType dt = es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                         : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = enc(m, dt, 5, t.ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename Kernel>
attn_status_t set_smem(Kernel k, int bytes) {
  // cudaFuncSetAttribute is cheap and idempotent; the result is per device.
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

attn_status_t last_launch() {
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Streaming multiprocessors of the current device (148 on a B200).
int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

// ---------------------------------------------------------------- forward
template <typename T, int D, int BC, int NS>
attn_status_t launch_single(const attn_tensor_t& q, const attn_tensor_t& k, const attn_tensor_t& v,
                            const eta::FwdParams& p, int B, int Hq, int Hkv, int N,
                            cudaStream_t st) {
  using C = eta::SingleCfg<T, D, BC, NS>;
  CUtensorMap tq, tk, tv;
  attn_status_t s;
  // whole-tile boxes: one TMA instruction per Q tile and per K or V tile
  if ((s = make_tile_map(&tq, q, B, Hq, N, D, sizeof(T), 128, C::NCHUNK)) != ATTN_OK) return s;
  if ((s = make_tile_map(&tk, k, B, Hkv, N, D, sizeof(T), BC, C::NCHUNK)) != ATTN_OK) return s;
  if ((s = make_tile_map(&tv, v, B, Hkv, N, D, sizeof(T), BC, C::NCHUNK)) != ATTN_OK) return s;
  auto kern = p.bmask ? eta::fwd_single_kernel<T, D, BC, NS, true>
                      : eta::fwd_single_kernel<T, D, BC, NS, false>;
  if ((s = set_smem(kern, C::SMEM_BYTES)) != ATTN_OK) return s;
  const unsigned tiles = static_cast<unsigned>((N + 127) / 128);
  const dim3 grid = p.head_major ? dim3(tiles, Hq, B) : dim3(Hq, B, tiles);
  CUtensorMap to;  // O as [B, Hq, N, D] bf16 ({64, 32} boxes) for TMA-store epilogues
  const attn_tensor_t o_t{p.o, p.osb, p.osh, p.osn};
  if ((s = make_map(&to, o_t, B, Hq, N, D, 2, 32)) != ATTN_OK) return s;
  kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tq, tk, tv, to, p);
  return last_launch();
}

// CTA pairs (tcgen05 .cta_group::2): two query heads of one GQA group when
// the group size is even, else two adjacent query tiles of one head; a
// cluster of two CTAs per pair.
template <int D, int BC, int NS>
attn_status_t launch_pair(const attn_tensor_t& q, const attn_tensor_t& k, const attn_tensor_t& v,
                          const eta::FwdParams& p, int B, int Hq, int Hkv, int N,
                          cudaStream_t st) {
  using C = eta::PairCfg<D, BC, NS>;
  CUtensorMap tq, tk, tv, to;
  attn_status_t s;
  if ((s = make_tile_map(&tq, q, B, Hq, N, D, 2, 128, C::NCHUNK)) != ATTN_OK) return s;
  // this CTA's half of a K tile: BC/2 rows, every chunk; of a V tile: every
  // row, half of the chunks
  if ((s = make_tile_map(&tk, k, B, Hkv, N, D, 2, C::KROWS, C::NCHUNK)) != ATTN_OK) return s;
  if ((s = make_tile_map(&tv, v, B, Hkv, N, D, 2, BC, C::VCH)) != ATTN_OK) return s;
  const attn_tensor_t o_t{p.o, p.osb, p.osh, p.osn};
  if ((s = make_map(&to, o_t, B, Hq, N, D, 2, 32)) != ATTN_OK) return s;
  auto kern = eta::fwd_pair_kernel<D, BC, NS>;
  if ((s = set_smem(kern, C::SMEM_BYTES)) != ATTN_OK) return s;
  const int tiles = (N + 127) / 128;
  const int heads_paired = (Hq / Hkv) % 2 == 0 ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = heads_paired ? dim3(Hq, B, tiles) : dim3(2 * Hq, B, (tiles + 1) / 2);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, p, heads_paired) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return last_launch();
}

// ---------------------------------------------------------------- backward
template <int D, int NQS, int NPB>
attn_status_t launch_bwd(const attn_tensor_t& q, const attn_tensor_t& k, const attn_tensor_t& v,
                         const attn_tensor_t& dout, eta::BwdParams& p, cudaStream_t st) {
  using C = eta::BwdCfg<D, NQS, NPB>;
  CUtensorMap tq, tk, tv, tdo;
  attn_status_t s;
  if ((s = make_map(&tq, q, p.B, p.Hq, p.N, D, 2, C::BR)) != ATTN_OK) return s;
  if ((s = make_map(&tdo, dout, p.B, p.Hq, p.N, D, 2, C::BR)) != ATTN_OK) return s;
  if ((s = make_map(&tk, k, p.B, p.Hkv, p.N, D, 2, C::BC)) != ATTN_OK) return s;
  if ((s = make_map(&tv, v, p.B, p.Hkv, p.N, D, 2, C::BC)) != ATTN_OK) return s;
  // fp32 dQ scratch as a (D, N, B*Hq) tensor; boxes of 32 columns x 64 rows
  CUtensorMap tdq;
  {
    auto enc = encode_fn();
    if (!enc) return ATTN_ERR_CUDA;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(p.N),
                          static_cast<cuuint64_t>(p.B) * p.Hq};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4,
                             static_cast<cuuint64_t>(D) * 4 * p.N};
    cuuint32_t box[3] = {32u, static_cast<cuuint32_t>(C::BR), 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    if (enc(&tdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.dqacc, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return ATTN_ERR_CUDA;
  }
  const long long rows = static_cast<long long>(p.B) * p.Hq * p.Npad;
  eta::bwd_preprocess_kernel<D><<<static_cast<unsigned>((rows / eta::kPrepRows * (D / 8) + 255) / 256), 256, 0, st>>>(p);
  if ((s = last_launch()) != ATTN_OK) return s;
  auto kern = eta::bwd_dkdv_kernel<D, NQS, NPB>;
  if ((s = set_smem(kern, C::SMEM_BYTES)) != ATTN_OK) return s;
  dim3 grid(p.Hkv * C::DSPLIT, p.B, (p.N + C::BC - 1) / C::BC);
  cudaEvent_t ev0 = static_cast<cudaEvent_t>(g_bwd_ev_start.exchange(nullptr));
  cudaEvent_t ev1 = static_cast<cudaEvent_t>(g_bwd_ev_stop.exchange(nullptr));
  g_bwd_q_ev_start.store(nullptr);  // this form has no separate dQ kernel
  g_bwd_q_ev_stop.store(nullptr);
  const bool timed = ev0 && ev1;
  if (timed && cudaEventRecord(ev0, st) != cudaSuccess) return ATTN_ERR_CUDA;
  kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tq, tk, tv, tdo, tdq, p);
  if ((s = last_launch()) != ATTN_OK) return s;
  if (timed && cudaEventRecord(ev1, st) != cudaSuccess) return ATTN_ERR_CUDA;
  const long long vec = static_cast<long long>(p.B) * p.Hq * p.N * (D / 8);
  eta::bwd_dq_finalize_kernel<D><<<static_cast<unsigned>((vec + 255) / 256), 256, 0, st>>>(p);
  return last_launch();
}

// Head dimensions 64 and 128: preprocess, then the column-parallel dK/dV
// kernel and the row-parallel dQ kernel (no scratch, no atomics).  With DS
// (D = 128, p.ds set) the dK/dV kernel also stores every visible dS^T tile and
// the dQ kernel sums dS K_j from them (bwd_dqs.cuh) instead of recomputing.
template <int D, int NQS, int NK, int NV, int NWG, bool DS = false>
attn_status_t launch_bwd_split(const attn_tensor_t& q, const attn_tensor_t& k,
                               const attn_tensor_t& v, const attn_tensor_t& dout,
                               eta::BwdParams& p, cudaStream_t st) {
  // D = 128: the dK/dV kernel with three Q stages (P^T in tensor memory)
  constexpr bool kKV3 = D == 128 && ETA_KV3;
  static_assert(!DS || kKV3, "stored dS tiles come from the three-stage dK/dV kernel");
  using CKV = eta::BwdKVCfg<D, NQS, NWG>;
  using CKV3 = eta::BwdKV3Cfg<128, 3, 2, 2>;
  using CQ = eta::BwdQCfg<D, NK, NV, NWG>;
  using CQS = eta::BwdDqsCfg<3>;
  CUtensorMap tq, tk, tv, tdo;
  attn_status_t s;
  if ((s = make_map(&tq, q, p.B, p.Hq, p.N, D, 2, 128)) != ATTN_OK) return s;
  if ((s = make_map(&tdo, dout, p.B, p.Hq, p.N, D, 2, 128)) != ATTN_OK) return s;
  if ((s = make_map(&tk, k, p.B, p.Hkv, p.N, D, 2, 128)) != ATTN_OK) return s;
  if ((s = make_map(&tv, v, p.B, p.Hkv, p.N, D, 2, 128)) != ATTN_OK) return s;
  const long long rows = static_cast<long long>(p.B) * p.Hq * p.Npad;
  eta::bwd_preprocess_kernel<D><<<static_cast<unsigned>((rows / eta::kPrepRows * (D / 8) + 255) / 256), 256, 0, st>>>(p);
  if ((s = last_launch()) != ATTN_OK) return s;
  auto kkv = kKV3 ? eta::bwd_kv3_kernel<128, 3, 2, 2, DS> : eta::bwd_kv_kernel<D, NQS, NWG>;
  const int kv_smem = kKV3 ? CKV3::SMEM_BYTES : CKV::SMEM_BYTES;
  const int kv_threads = kKV3 ? CKV3::THREADS : CKV::THREADS;
  auto kq = eta::bwd_q_kernel<D, NK, NV, NWG>;
  auto kqs = eta::bwd_dqs_kernel<3>;
  if ((s = set_smem(kkv, kv_smem)) != ATTN_OK) return s;
  if (DS) {
    if ((s = set_smem(kqs, CQS::SMEM_BYTES)) != ATTN_OK) return s;
  } else {
    if ((s = set_smem(kq, CQ::SMEM_BYTES)) != ATTN_OK) return s;
  }
  const unsigned tiles = static_cast<unsigned>((p.N + 127) / 128);
  cudaEvent_t ev0 = static_cast<cudaEvent_t>(g_bwd_ev_start.exchange(nullptr));
  cudaEvent_t ev1 = static_cast<cudaEvent_t>(g_bwd_ev_stop.exchange(nullptr));
  const bool timed = ev0 && ev1;
  if (timed && cudaEventRecord(ev0, st) != cudaSuccess) return ATTN_ERR_CUDA;
  // persistent: one CTA per SM (at most one per work item)
  const long long kv_items = static_cast<long long>(p.Hkv) * p.B * tiles;
  const unsigned kv_ctas = static_cast<unsigned>(std::min<long long>(kv_items, sm_count()));
  // dK, dV as [B, Hkv, N, D] for the TMA stores of the epilogue ({64, 32} boxes)
  CUtensorMap tdk, tdv;
  const attn_tensor_t dk_t{p.dk, p.dksb, p.dksh, p.dksn}, dv_t{p.dv, p.dvsb, p.dvsh, p.dvsn};
  if ((s = make_map(&tdk, dk_t, p.B, p.Hkv, p.N, D, 2, 32)) != ATTN_OK) return s;
  if ((s = make_map(&tdv, dv_t, p.B, p.Hkv, p.N, D, 2, 32)) != ATTN_OK) return s;
  kkv<<<kv_ctas, kv_threads, kv_smem, st>>>(tq, tk, tv, tdo, tdk, tdv, p);
  if ((s = last_launch()) != ATTN_OK) return s;
  if (timed && cudaEventRecord(ev1, st) != cudaSuccess) return ATTN_ERR_CUDA;
  CUtensorMap tdq;
  const attn_tensor_t dq_t{p.dq, p.dqsb, p.dqsh, p.dqsn};
  if ((s = make_map(&tdq, dq_t, p.B, p.Hq, p.N, D, 2, 32)) != ATTN_OK) return s;
  cudaEvent_t eq0 = static_cast<cudaEvent_t>(g_bwd_q_ev_start.exchange(nullptr));
  cudaEvent_t eq1 = static_cast<cudaEvent_t>(g_bwd_q_ev_stop.exchange(nullptr));
  const bool qtimed = eq0 && eq1;
  if (qtimed && cudaEventRecord(eq0, st) != cudaSuccess) return ATTN_ERR_CUDA;
  const dim3 qgrid = p.head_major ? dim3(tiles, p.Hq, p.B) : dim3(p.Hq, p.B, tiles);
  // programmatic dependent launch: the dQ kernel's CTAs take the SMs the
  // persistent dK/dV CTAs leave as they finish (the seven-product one reads
  // nothing they write; the stored-dS one waits for their completion before
  // its first read of the tiles); an event recorded in between (the timing
  // hook) serialises the two
  cudaLaunchConfig_t cfg = {};
  // the stored-dS dQ kernel is persistent: one CTA per SM (at most one per query tile)
  const long long q_items = static_cast<long long>(p.Hq) * p.B * tiles;
  cfg.gridDim = DS ? dim3(static_cast<unsigned>(std::min<long long>(q_items, sm_count())), 1, 1)
                   : qgrid;
  cfg.blockDim = dim3(DS ? CQS::THREADS : CQ::THREADS, 1, 1);
  cfg.dynamicSmemBytes = DS ? CQS::SMEM_BYTES : CQ::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t le = DS ? cudaLaunchKernelEx(&cfg, kqs, tk, tdq, p)
                            : cudaLaunchKernelEx(&cfg, kq, tq, tk, tv, tdo, tdq, p);
  if (le != cudaSuccess) return ATTN_ERR_CUDA;
  if ((s = last_launch()) != ATTN_OK) return s;
  if (qtimed && cudaEventRecord(eq1, st) != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

// ---------------------------------------------------------------- decode
constexpr int kDecodeMaxSplits = 64;
#ifndef ETA_DECODE_CTAS_PER_SM
#define ETA_DECODE_CTAS_PER_SM 4
#endif
constexpr long long kDecodeCtasPerSm = ETA_DECODE_CTAS_PER_SM;

// Splits of the page range per (sequence, key/value head): enough CTAs for
// about four per SM (in waves of one CTA per SM: fewer left a long tail,
// measured), at most one per page and kDecodeMaxSplits.
int decode_splits(int B, int Hkv, int max_pages, int* pages_per_split) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long units = static_cast<long long>(B) * Hkv;
  int splits = static_cast<int>(
      std::min<long long>(kDecodeMaxSplits, (kDecodeCtasPerSm * sms + units - 1) / units));
  splits = std::max(1, std::min(splits, max_pages));
  const int pps = (max_pages + splits - 1) / splits;
  *pages_per_split = pps;
  return (max_pages + pps - 1) / pps;
}

size_t decode_workspace(int B, int Hq, int Sq, int D, int max_pages) {
  const size_t rows = static_cast<size_t>(B) * Hq * Sq * std::min(max_pages, kDecodeMaxSplits);
  return eta::round_up(rows * D * 4, 256) + eta::round_up(rows * 4, 256);
}

// Page pool [P, 128, Hkv, D] (t.sb: page stride, t.sh: head stride, t.sn: row
// stride, in elements) as a 4-D TMA map over (D, Hkv, 128 rows, P) with
// boxes of 64 columns x 128 rows of one head.
attn_status_t make_pool_map(CUtensorMap* m, const attn_tensor_t& t, int P, int Hkv, int D) {
  auto enc = encode_fn();
  if (!enc) return ATTN_ERR_CUDA;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv), 128u,
                        static_cast<cuuint64_t>(P)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(t.sh) * 2, static_cast<cuuint64_t>(t.sn) * 2,
                           static_cast<cuuint64_t>(t.sb) * 2};
  cuuint32_t box[4] = {64u, 1u, 128u, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t.ptr, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t check_pool(const attn_tensor_t& t, int P, int Hkv) {
  if (!t.ptr) return ATTN_ERR_INVALID_ARG;
  if ((P > 1 && t.sb <= 0) || (Hkv > 1 && t.sh <= 0) || t.sn <= 0) return ATTN_ERR_INVALID_ARG;
  if (t.sb < 0 || t.sh < 0) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(t.ptr)) return ATTN_ERR_MISALIGNED;
  if ((t.sb * 2) % 16 || (t.sh * 2) % 16 || (t.sn * 2) % 16) return ATTN_ERR_MISALIGNED;
  return ATTN_OK;
}

template <int D, int NS>
attn_status_t launch_decode(const attn_tensor_t& kp, const attn_tensor_t& vp, int P,
                            eta::DecodeParams& p, cudaStream_t st) {
  using C = eta::DecodeCfg<D, NS>;
  CUtensorMap tk, tv;
  attn_status_t s;
  if ((s = make_pool_map(&tk, kp, P, p.Hkv, D)) != ATTN_OK) return s;
  if ((s = make_pool_map(&tv, vp, P, p.Hkv, D)) != ATTN_OK) return s;
  auto kern = eta::decode_kernel<D, NS>;
  if ((s = set_smem(kern, C::SMEM_BYTES)) != ATTN_OK) return s;
  kern<<<dim3(p.splits, p.Hkv, p.B), C::THREADS, C::SMEM_BYTES, st>>>(tk, tv, p);
  if ((s = last_launch()) != ATTN_OK) return s;
  const long long rows = static_cast<long long>(p.B) * p.Hq * p.Sq;
  eta::decode_combine_kernel<D><<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, st>>>(p);
  return last_launch();
}

// Grid order of the kernels with one CTA per query tile (forward, dQ): a
// head's query tiles together when every tile does about the same work (no
// block mask, and no key range that grows with the query index as under the
// causal mask), else the longest tiles of every head first.  Measured on B200:
// the 4x16x2048 non-causal forward 0.1505 -> 0.1413 ms head-major, the
// 2x16x4096 causal one 0.136 -> 0.165 ms (the late start of each head's
// longest tile leaves a tail).
int grid_head_major(int wl, int wr, const uint8_t* block_mask) {
  if (block_mask) return 0;
  return (wl < 0 && wr >= 0) ? 0 : 1;
}

attn_status_t check_sizes(int B, int Hq, int Hkv, int N) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (B > 65535 || Hq > 65535 || (N + 63) / 64 > 65535) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_abi_version(void) { return ATTN_ABI_VERSION; }

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ATTN_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
    case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

void attn_debug_set_wait_limit_ns(unsigned long long ns) {
  g_wait_limit_ns.store(ns ? ns : kDefaultWaitLimitNs);
}

void attn_debug_set_flags(int flags) { g_debug_flags.store(flags); }

void attn_debug_set_fwd_variant(int variant) {
  g_fwd_variant.store(variant >= 0 && variant <= 2 ? variant : 0);
}

void attn_debug_set_bwd_events(void* start, void* stop) {
  g_bwd_ev_start.store(start);
  g_bwd_ev_stop.store(stop);
}

void attn_debug_set_bwd_q_events(void* start, void* stop) {
  g_bwd_q_ev_start.store(start);
  g_bwd_q_ev_stop.store(stop);
}

#ifdef ETA_TRACE
ATTN_API int attn_debug_read_ftrace(void* dst, size_t bytes) {
  if (bytes > sizeof(eta::g_eta_ftrace)) bytes = sizeof(eta::g_eta_ftrace);
  return cudaMemcpyFromSymbol(dst, eta::g_eta_ftrace, bytes) == cudaSuccess ? 0 : 1;
}
ATTN_API int attn_debug_read_trace(void* dst, size_t bytes) {
  if (bytes > sizeof(eta::g_eta_trace)) bytes = sizeof(eta::g_eta_trace);
  return cudaMemcpyFromSymbol(dst, eta::g_eta_trace, bytes) == cudaSuccess ? 0 : 1;
}
#endif

attn_status_t attn_debug_exp2(const float* x, float* y, int n, int mode, void* stream) {
  if (!x || !y || n < 0 || (mode != 0 && mode != 1)) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  const int pairs = (n + 1) / 2;
  debug_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n,
                                                                                       mode);
  return last_launch();
}

attn_status_t attn_device_status(void* stream, int* where) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int host[4] = {0, 0, 0, 0};
  if (cudaMemcpyFromSymbol(host, g_attn_status, sizeof(host)) != cudaSuccess) return ATTN_ERR_CUDA;
  const int zero[4] = {0, 0, 0, 0};
  if (cudaMemcpyToSymbol(g_attn_status, zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (where) *where = host[1];
  if (host[0] == 0) return ATTN_OK;
  return host[0] == ATTN_ERR_DEVICE_TIMEOUT ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_ERR_CUDA;
}

attn_status_t attn_fwd(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v, attn_tensor_t o,
                       float* lse, int B, int Hq, int Hkv, int N, int D, attn_dtype_t dtype,
                       int causal, float scale, void* stream) {
  return attn_fwd_window(q, k, v, o, lse, B, Hq, Hkv, N, D, dtype, -1, causal ? 0 : -1, scale,
                         stream);
}

attn_status_t attn_fwd_window(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v, attn_tensor_t o,
                              float* lse, int B, int Hq, int Hkv, int N, int D,
                              attn_dtype_t dtype, int window_left, int window_right, float scale,
                              void* stream) {
  return attn_fwd_masked(q, k, v, o, lse, B, Hq, Hkv, N, D, dtype, window_left, window_right,
                         nullptr, scale, stream);
}

attn_status_t attn_fwd_masked(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v, attn_tensor_t o,
                              float* lse, int B, int Hq, int Hkv, int N, int D,
                              attn_dtype_t dtype, int window_left, int window_right,
                              const uint8_t* block_mask, float scale, void* stream) {
  attn_status_t s;
  if (window_left < -1 || window_right < -1) return ATTN_ERR_INVALID_ARG;
  if ((s = check_sizes(B, Hq, Hkv, N)) != ATTN_OK) return s;
  if (!lse) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP32) return ATTN_ERR_INVALID_ARG;
  const bool bf16 = dtype == ATTN_BF16;
  if (bf16 ? !(D == 64 || D == 128 || D == 256) : D != 64) return ATTN_ERR_UNSUPPORTED;
  if (block_mask) {
    // block-sparse tiles: bf16 with D <= 128 and at most kMaxMaskTiles tiles
    if (!bf16 || D > 128 || (N + 127) / 128 > eta::kMaxMaskTiles) return ATTN_ERR_UNSUPPORTED;
  }
  const int es = bf16 ? 2 : 4;
  if ((s = check_tensor(q, B, Hq, N, es)) != ATTN_OK) return s;
  if ((s = check_tensor(k, B, Hkv, N, es)) != ATTN_OK) return s;
  if ((s = check_tensor(v, B, Hkv, N, es)) != ATTN_OK) return s;
  if ((s = check_tensor(o, B, Hq, N, es)) != ATTN_OK) return s;
  if ((s = check_output_layout(o, B, Hq, N, D)) != ATTN_OK) return s;
  if (!aligned16(lse)) return ATTN_ERR_MISALIGNED;

  eta::FwdParams p;
  p.o = o.ptr;
  p.lse = lse;
  p.osb = o.sb;
  p.osh = o.sh;
  p.osn = o.sn;
  p.Hq = Hq;
  p.N = N;
  p.group = Hq / Hkv;
  p.wl = window_left >= N ? -1 : window_left;
  p.wr = window_right >= N ? -1 : window_right;
  p.scale = scale;
  p.c = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  if ((s = status_ptr(&p.status)) != ATTN_OK) return s;
  p.wait_limit_ns = g_wait_limit_ns.load();
  p.debug_flags = g_debug_flags.load();
  p.o_mul = 1.f;
  p.bmask = block_mask;
  p.nt = (N + 127) / 128;
  p.head_major = grid_head_major(p.wl, p.wr, block_mask);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!bf16) {
    dim3 grid((N + eta::kF32Rows - 1) / eta::kF32Rows, Hq, B);
    eta::fwd_fp32_kernel<<<grid, 128, 0, st>>>(
        static_cast<const float*>(q.ptr), static_cast<const float*>(k.ptr),
        static_cast<const float*>(v.ptr), q.sb, q.sh, q.sn, k.sb, k.sh, k.sn, v.sb, v.sh, v.sn, p);
    return last_launch();
  }
  // One query tile per CTA with 64-key tiles and a double-buffered S; at
  // D <= 128 two CTAs share an SM (faster than the two-tile ping-pong CTA,
  // measured: each CTA's S(j+1) runs while its softmax of S(j) does, and one
  // CTA's loads and epilogue overlap the other's products).
  switch (D) {
    case 64: return launch_single<__nv_bfloat16, 64, 64, 8>(q, k, v, p, B, Hq, Hkv, N, st);
    case 128:
      if (!block_mask && g_fwd_variant.load() == 2)
        return launch_pair<128, 64, 8>(q, k, v, p, B, Hq, Hkv, N, st);
      return launch_single<__nv_bfloat16, 128, 64, 4>(q, k, v, p, B, Hq, Hkv, N, st);
    default: return launch_single<__nv_bfloat16, 256, 64, 4>(q, k, v, p, B, Hq, Hkv, N, st);
  }
}

attn_status_t attn_fwd_fp8(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v, attn_tensor_t o,
                           float* lse, int B, int Hq, int Hkv, int N, int D, float q_scale,
                           float k_scale, float v_scale, int window_left, int window_right,
                           float scale, void* stream) {
  attn_status_t s;
  if (window_left < -1 || window_right < -1) return ATTN_ERR_INVALID_ARG;
  if ((s = check_sizes(B, Hq, Hkv, N)) != ATTN_OK) return s;
  if (!lse) return ATTN_ERR_INVALID_ARG;
  for (float f : {scale, q_scale, k_scale, v_scale})
    if (!(f > 0.f) || !std::isfinite(f)) return ATTN_ERR_INVALID_ARG;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  if ((s = check_tensor(q, B, Hq, N, 1)) != ATTN_OK) return s;
  if ((s = check_tensor(k, B, Hkv, N, 1)) != ATTN_OK) return s;
  if ((s = check_tensor(v, B, Hkv, N, 1)) != ATTN_OK) return s;
  if ((s = check_tensor(o, B, Hq, N, 2)) != ATTN_OK) return s;
  if ((s = check_output_layout(o, B, Hq, N, D)) != ATTN_OK) return s;
  if (!aligned16(lse)) return ATTN_ERR_MISALIGNED;
  eta::FwdParams p;
  p.o = o.ptr;
  p.lse = lse;
  p.osb = o.sb;
  p.osh = o.sh;
  p.osn = o.sn;
  p.Hq = Hq;
  p.N = N;
  p.group = Hq / Hkv;
  p.wl = window_left >= N ? -1 : window_left;
  p.wr = window_right >= N ? -1 : window_right;
  // the per-tensor scales fold into the score scale and the output multiplier
  const double se = static_cast<double>(scale) * q_scale * k_scale;
  p.scale = static_cast<float>(se);
  p.c = static_cast<float>(se * 1.4426950408889634);
  if (!std::isfinite(p.c) || !(p.scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if ((s = status_ptr(&p.status)) != ATTN_OK) return s;
  p.wait_limit_ns = g_wait_limit_ns.load();
  p.debug_flags = 0;
  p.o_mul = v_scale / eta::kP8Scale;
  p.bmask = nullptr;
  p.nt = (N + 127) / 128;
  p.head_major = grid_head_major(p.wl, p.wr, nullptr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return launch_single<__nv_fp8_e4m3, 128, 64, 8>(q, k, v, p, B, Hq, Hkv, N, st);
}

size_t attn_decode_workspace_bytes(int B, int Hq, int Sq, int D, int max_pages) {
  if (B < 1 || Hq < 1 || Sq < 1 || D < 1 || max_pages < 1) return 0;
  return decode_workspace(B, Hq, Sq, D, max_pages);
}

attn_status_t attn_decode_paged(attn_tensor_t q, attn_tensor_t k_pool, attn_tensor_t v_pool,
                                int num_pages, const int* block_table, int max_pages,
                                const int* seqlens, attn_tensor_t o, float* lse, int B, int Hq,
                                int Hkv, int Sq, int D, attn_dtype_t dtype, int causal,
                                float scale, void* workspace, size_t workspace_bytes,
                                void* stream) {
  attn_status_t s;
  if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || num_pages < 1 || max_pages < 1)
    return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!block_table || !seqlens || !lse) return ATTN_ERR_INVALID_ARG;
  if (!workspace) return ATTN_ERR_WORKSPACE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_BF16) return dtype == ATTN_FP32 ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
  if (!(D == 64 || D == 128)) return ATTN_ERR_UNSUPPORTED;
  if ((Hq / Hkv) * Sq > 128 || B > 65535 || Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
  if ((s = check_tensor(q, B, Hq, Sq, 2)) != ATTN_OK) return s;
  if ((s = check_tensor(o, B, Hq, Sq, 2)) != ATTN_OK) return s;
  if ((s = check_output_layout(o, B, Hq, Sq, D)) != ATTN_OK) return s;
  if ((s = check_pool(k_pool, num_pages, Hkv)) != ATTN_OK) return s;
  if ((s = check_pool(v_pool, num_pages, Hkv)) != ATTN_OK) return s;
  if (!aligned16(lse)) return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < decode_workspace(B, Hq, Sq, D, max_pages)) return ATTN_ERR_WORKSPACE;
  eta::DecodeParams p;
  p.q = q.ptr;
  p.qsb = q.sb; p.qsh = q.sh; p.qsn = q.sn;
  p.o = o.ptr;
  p.osb = o.sb; p.osh = o.sh; p.osn = o.sn;
  p.lse = lse;
  p.block_table = block_table;
  p.seqlens = seqlens;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Sq = Sq; p.group = Hq / Hkv;
  p.max_pages = max_pages;
  p.splits = decode_splits(B, Hkv, max_pages, &p.pages_per_split);
  const size_t rows = static_cast<size_t>(B) * Hq * Sq * p.splits;
  p.part_o = static_cast<float*>(workspace);
  p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                        eta::round_up(rows * D * 4, 256));
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.c = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  if ((s = status_ptr(&p.status)) != ATTN_OK) return s;
  p.wait_limit_ns = g_wait_limit_ns.load();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 64) return launch_decode<64, 8>(k_pool, v_pool, num_pages, p, st);
  return launch_decode<128, 6>(k_pool, v_pool, num_pages, p, st);
}

size_t attn_bwd_workspace_bytes(int B, int Hq, int N, int D) {
  if (B < 1 || Hq < 1 || N < 1 || D < 1) return 0;
  return eta::bwd_workspace_bytes(B, Hq, N, D);
}

size_t attn_bwd_workspace_bytes_ds(int B, int Hq, int N, int D, int window_left,
                                   int window_right) {
  if (B < 1 || Hq < 1 || N < 1 || D < 1 || window_left < -1 || window_right < -1) return 0;
  const int wl = window_left >= N ? -1 : window_left, wr = window_right >= N ? -1 : window_right;
  const size_t ds = eta::ds_bytes(B, Hq, N, D, wl, wr);
  if (ds == 0) return eta::bwd_workspace_bytes(B, Hq, N, D);
  return eta::ds_offset(B, Hq, N, D) + ds;
}

attn_status_t attn_bwd(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v, attn_tensor_t o,
                       const float* lse, attn_tensor_t dout, attn_tensor_t dq, attn_tensor_t dk,
                       attn_tensor_t dv, int B, int Hq, int Hkv, int N, int D,
                       attn_dtype_t dtype, int causal, float scale, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return attn_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, D, dtype, -1,
                         causal ? 0 : -1, scale, workspace, workspace_bytes, stream);
}

attn_status_t attn_bwd_window(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v, attn_tensor_t o,
                              const float* lse, attn_tensor_t dout, attn_tensor_t dq,
                              attn_tensor_t dk, attn_tensor_t dv, int B, int Hq, int Hkv, int N,
                              int D, attn_dtype_t dtype, int window_left, int window_right,
                              float scale, void* workspace, size_t workspace_bytes,
                              void* stream) {
  return attn_bwd_masked(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, D, dtype, window_left,
                         window_right, nullptr, scale, workspace, workspace_bytes, stream);
}

attn_status_t attn_bwd_masked(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v, attn_tensor_t o,
                              const float* lse, attn_tensor_t dout, attn_tensor_t dq,
                              attn_tensor_t dk, attn_tensor_t dv, int B, int Hq, int Hkv, int N,
                              int D, attn_dtype_t dtype, int window_left, int window_right,
                              const uint8_t* block_mask, float scale, void* workspace,
                              size_t workspace_bytes, void* stream) {
  attn_status_t s;
  if (window_left < -1 || window_right < -1) return ATTN_ERR_INVALID_ARG;
  if ((s = check_sizes(B, Hq, Hkv, N)) != ATTN_OK) return s;
  if (!lse || !workspace) return !lse ? ATTN_ERR_INVALID_ARG : ATTN_ERR_WORKSPACE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_BF16) return dtype == ATTN_FP32 ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
  if (!(D == 64 || D == 128 || D == 256)) return ATTN_ERR_UNSUPPORTED;
  if (block_mask && (D > 128 || (N + 127) / 128 > eta::kMaxMaskTiles)) return ATTN_ERR_UNSUPPORTED;
  const int es = 2;
  const attn_tensor_t* qs[] = {&q, &o, &dout, &dq};
  for (auto* t : qs)
    if ((s = check_tensor(*t, B, Hq, N, es)) != ATTN_OK) return s;
  const attn_tensor_t* ks[] = {&k, &v, &dk, &dv};
  for (auto* t : ks)
    if ((s = check_tensor(*t, B, Hkv, N, es)) != ATTN_OK) return s;
  if ((s = check_output_layout(dq, B, Hq, N, D)) != ATTN_OK) return s;
  if ((s = check_output_layout(dk, B, Hkv, N, D)) != ATTN_OK) return s;
  if ((s = check_output_layout(dv, B, Hkv, N, D)) != ATTN_OK) return s;
  if (!aligned16(lse)) return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < eta::bwd_workspace_bytes(B, Hq, N, D)) return ATTN_ERR_WORKSPACE;
  eta::BwdParams p;
  p.o = o.ptr;
  p.dout = dout.ptr;
  p.lse = lse;
  p.dq = dq.ptr;
  p.dk = dk.ptr;
  p.dv = dv.ptr;
  char* ws = static_cast<char*>(workspace);
  p.dqacc = eta::bwd_dqacc_bytes(B, Hq, N, D) ? reinterpret_cast<float*>(ws) : nullptr;
  p.delta = reinterpret_cast<float*>(ws + eta::bwd_dqacc_bytes(B, Hq, N, D));
  p.lse2 = reinterpret_cast<float*>(ws + eta::bwd_dqacc_bytes(B, Hq, N, D) +
                                    eta::bwd_stat_bytes(B, Hq, N));
  p.osb = o.sb; p.osh = o.sh; p.osn = o.sn;
  p.dosb = dout.sb; p.dosh = dout.sh; p.dosn = dout.sn;
  p.dqsb = dq.sb; p.dqsh = dq.sh; p.dqsn = dq.sn;
  p.dksb = dk.sb; p.dksh = dk.sh; p.dksn = dk.sn;
  p.dvsb = dv.sb; p.dvsh = dv.sh; p.dvsn = dv.sn;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.N = N; p.D = D;
  p.Npad = static_cast<int>(eta::bwd_npad(N));
  p.group = Hq / Hkv;
  p.wl = window_left >= N ? -1 : window_left;
  p.wr = window_right >= N ? -1 : window_right;
  p.scale = scale;
  p.c = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  if ((s = status_ptr(&p.status)) != ATTN_OK) return s;
  p.wait_limit_ns = g_wait_limit_ns.load();
  p.bmask = block_mask;
  p.nt = (N + 127) / 128;
  p.debug_flags = g_debug_flags.load();
  p.head_major = grid_head_major(p.wl, p.wr, block_mask);
  // stored dS tiles when the workspace holds them (head dimension 128)
  p.ds = nullptr;
  p.ds_head = 0;
  p.ds_tri = 0;
  p.ds_w = 0;
  const size_t ds_need = ETA_KV3 ? eta::ds_bytes(B, Hq, N, D, p.wl, p.wr) : 0;
  if (ds_need > 0 && workspace_bytes >= eta::ds_offset(B, Hq, N, D) + ds_need) {
    p.ds = reinterpret_cast<uint8_t*>(ws + eta::ds_offset(B, Hq, N, D));
    eta::ds_layout(N, p.wl, p.wr, &p.ds_tri, &p.ds_w, &p.ds_head);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // per head dimension: Q/dO stages of the dK/dV kernel, K and V ring slots
  // of the dQ kernel, elementwise warpgroups (measured best on B200)
  if (D == 64) return launch_bwd_split<64, 4, 5, 3, 4>(q, k, v, dout, p, st);
  if (D == 128 && p.ds) return launch_bwd_split<128, 2, 3, 2, 2, true>(q, k, v, dout, p, st);
  if (D == 128) return launch_bwd_split<128, 2, 3, 2, 2>(q, k, v, dout, p, st);
  return launch_bwd<256, 1, 1>(q, k, v, dout, p, st);
}

}  // extern "C"

// ---------------------------------------------------------------- backward without allocation
// Fixed scratch used by attn_bwd_noalloc in place of a caller-provided
// workspace.  In host code the name below is only a host-side stand-in for
// the array; its device address comes from cudaGetSymbolAddress, once per
// device, with that device current.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_noalloc_ptr[kMaxDevices] = {};

attn_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ATTN_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" attn_status_t attn_bwd_noalloc(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v,
                                          attn_tensor_t o, const float* lse, attn_tensor_t dout,
                                          attn_tensor_t dq, attn_tensor_t dk, attn_tensor_t dv,
                                          int B, int Hq, int Hkv, int N, int D,
                                          attn_dtype_t dtype, int causal, float scale,
                                          void* stream) {
  const size_t need = attn_bwd_workspace_bytes(B, Hq, N, D);
  if (need == 0) return ATTN_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return ATTN_ERR_WORKSPACE;  // beyond the fixed scratch
  void* ws = nullptr;
  attn_status_t s = noalloc_scratch(&ws);
  if (s != ATTN_OK) return s;
  return attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, D, dtype, causal, scale, ws,
                  kNoAllocScratchBytes, stream);
}
