/*
 * Exact tiled attention for NVIDIA B200 (sm_100a) -- C ABI.
 *
 * The operation (r/mlscaling, FlashAttention-PyTorch post: every generation
 * FA1..FA4 keeps "the same exact attention math"; FlashAttention entity
 * page, finding "FlashAttention-4: Algorithm and Kernel Pipelining for
 * Blackwell GPUs"; FlashAttention (Metal Port) README, Documentation section,
 * for the recompute-based backward with its scratch for atomics and partial
 * sums):
 *
 *   forward   S = scale * Q K^T, S[i][j] = -inf for j > i when causal,
 *             P = row-softmax(S), O = P V, lse[i] = ln(sum_j exp(S[i][j]))
 *   backward  dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dO * O)),
 *             dQ = scale dS K, dK = scale dS^T Q, with P recomputed from lse
 *
 * Grouped-query attention: query head h reads key/value head h / (Hq / Hkv)
 * (contiguous groups); dK and dV sum over the group.
 *
 * Tensors.  Every Q/K/V/O/dO/dQ/dK/dV tensor is a 4-D [B, H, N, D] array
 * described by an attn_tensor_t: a device pointer and the element strides of
 * the B, H and N dimensions; the D dimension has unit stride.  H is Hq for
 * Q, O, dO, dQ and Hkv for K, V, dK, dV.  lse is a contiguous fp32
 * [B, Hq, N] device array.  All pointers are device pointers owned by the
 * caller; the library allocates no device memory and keeps no pointer after
 * a call returns.
 *
 * Requirements (checked before anything is launched; a violation returns an
 * error code and launches nothing):
 *   B, Hq, Hkv, N >= 1; Hq % Hkv == 0; D in {64, 128, 256};
 *   every pointer 16-byte aligned and every stride a multiple of 16 bytes
 *   (the tensor-memory-accelerator rule);
 *   ATTN_FP32 (fp32 storage, products and accumulation in fp32 on the CUDA
 *   cores, not the tensor cores) only for the forward with D = 64; the
 *   backward supports bf16 with D in {64, 128, 256};
 *   an output tensor must not overlap itself (with its dimensions sorted by
 *   stride, each stride must exceed the span of the dimensions inside it),
 *   else ATTN_ERR_INVALID_ARG.
 *
 * Every call is asynchronous on `stream` (a cudaStream_t, NULL = legacy
 * default stream).  The return value reports host-side validation and launch
 * errors only.  A kernel whose internal wait times out (it never hangs: each
 * wait is bounded) records ATTN_ERR_DEVICE_TIMEOUT in a device status word
 * that attn_device_status() reads.  There is one status word per device,
 * shared by every stream and host thread that calls the library on it: the
 * first failure since the last read is kept, and attn_device_status() on any
 * stream returns (and clears) it.  A caller that runs work on several streams
 * should synchronise all of them before reading it, so that the failure is
 * attributed to the right batch of calls.
 */
#ifndef EXACT_TILED_ATTENTION_ATTN_H_
#define EXACT_TILED_ATTENTION_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ATTN_ABI_VERSION 1

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

typedef struct attn_tensor {
  void* ptr;   /* device pointer to element [0, 0, 0, 0] */
  int64_t sb;  /* element stride of the batch dimension */
  int64_t sh;  /* element stride of the head dimension */
  int64_t sn;  /* element stride of the sequence dimension */
} attn_tensor_t;

typedef enum attn_dtype {
  ATTN_BF16 = 0, /* bf16 storage, fp32 accumulation */
  ATTN_FP32 = 1  /* fp32 storage, fp32 products and accumulation (CUDA cores) */
} attn_dtype_t;

typedef enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, Hq % Hkv != 0 */
  ATTN_ERR_UNSUPPORTED = 2,    /* head dim / dtype / direction not built */
  ATTN_ERR_MISALIGNED = 3,     /* pointer or stride breaks the 16-byte rule */
  ATTN_ERR_WORKSPACE = 4,      /* workspace missing or smaller than required */
  ATTN_ERR_CUDA = 5,           /* a CUDA runtime/driver call failed */
  ATTN_ERR_DEVICE_TIMEOUT = 6  /* a kernel's bounded wait gave up (device status) */
} attn_status_t;

/* ABI version of the loaded library (ATTN_ABI_VERSION). */
ATTN_API int attn_abi_version(void);

/* Human-readable name of a status code (static string). */
ATTN_API const char* attn_status_string(attn_status_t status);

/*
 * Forward.  Reads q [B,Hq,N,D], k and v [B,Hkv,N,D]; writes o [B,Hq,N,D]
 * (same dtype as the inputs) and lse [B,Hq,N] (fp32, natural log of the sum
 * of exp of the scaled, masked scores).  causal != 0 applies the top-left
 * causal mask (key j visible to query i iff j <= i).  scale multiplies
 * q.k (1/sqrt(D) is the usual choice).  o must not alias q, k or v.
 */
ATTN_API attn_status_t attn_fwd(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v, attn_tensor_t o,
                       float* lse, int B, int Hq, int Hkv, int N, int D, attn_dtype_t dtype,
                       int causal, float scale, void* stream);

/*
 * Forward with a local (sliding) window: query i sees key j only when
 * i - window_left <= j <= i + window_right; -1 leaves that side unbounded
 * (attn_fwd's causal mask is window (-1, 0), no mask is (-1, -1)).  Windows
 * wider than N behave as unbounded.  The pages name this mask variant: global
 * plus sliding-window attention (heapsort-ai.news attention tag) and a
 * 112-token local window (twiscan MHA search), i.e. window (111, 0).  Other
 * arguments as attn_fwd; window_left or window_right < -1 is
 * ATTN_ERR_INVALID_ARG.
 */
ATTN_API attn_status_t attn_fwd_window(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v,
                                       attn_tensor_t o, float* lse, int B, int Hq, int Hkv, int N,
                                       int D, attn_dtype_t dtype, int window_left,
                                       int window_right, float scale, void* stream);

/*
 * Forward with a window (as attn_fwd_window) and a block-sparse tile mask
 * (FlashAttention (Metal Port) README, Documentation section: block sparsity
 * as a customisation of the basic algorithm; FlashPrefill V2 finding on the
 * FlashAttention entity page: block-sparse prefill).
 *
 * block_mask: NULL (dense), or a device array of T x T bytes per (batch,
 * query head), [B][Hq][T][T] contiguous, T = ceil(N / 128): query i sees key
 * j only when block_mask[b][h][i / 128][j / 128] != 0 (and the window allows
 * it); tile pairs whose byte is 0 are skipped, not computed.  Owned by the
 * caller, read during the call's kernels only.  A query row that sees no key
 * gets o = 0 and lse = -inf.  With a mask: bf16 with D in {64, 128} and
 * T <= 512 (N <= 65536); anything else is ATTN_ERR_UNSUPPORTED.
 */
ATTN_API attn_status_t attn_fwd_masked(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v,
                                       attn_tensor_t o, float* lse, int B, int Hq, int Hkv, int N,
                                       int D, attn_dtype_t dtype, int window_left,
                                       int window_right, const uint8_t* block_mask, float scale,
                                       void* stream);

/*
 * Bytes of device workspace attn_bwd needs for these sizes: two fp32 row
 * statistics [B,Hq,N'] (rowsum(dO*O) and lse*log2(e), N' = N rounded up to
 * 128), and for D = 256 also an fp32 dQ accumulator [B,Hq,N,D] (the scratch
 * that backward's partial sums are added into).  Returns 0 for invalid sizes.
 */
ATTN_API size_t attn_bwd_workspace_bytes(int B, int Hq, int N, int D);

/*
 * Bytes of workspace with which attn_bwd (window_left = -1, window_right = 0
 * for causal, -1 otherwise), attn_bwd_window and attn_bwd_masked with this
 * window store dS: head dimension 128 only.  The dK/dV kernel then also
 * writes each visible 128 x 128 tile's dS (bf16, 32 KB per tile: N^2 / 2
 * bytes per (batch, query head) for the causal mask, up to 2 N^2 for other
 * windows) into the workspace, and dQ is summed from those tiles (one
 * product per tile pair) instead of being recomputed with S and dP (three
 * products per tile pair).  Both forms sum in a fixed order (no atomics) and
 * are bitwise reproducible.  Equals attn_bwd_workspace_bytes where the
 * stored form does not apply (D != 128, or more than 4 GiB of tiles); 0 for
 * invalid sizes or windows.  A smaller workspace (at least
 * attn_bwd_workspace_bytes) selects the recomputing form.
 */
ATTN_API size_t attn_bwd_workspace_bytes_ds(int B, int Hq, int N, int D, int window_left,
                                            int window_right);

/*
 * Backward.  Reads q, k, v, the forward's o and lse, and the upstream
 * gradient dout [B,Hq,N,D]; writes dq [B,Hq,N,D], dk and dv [B,Hkv,N,D]
 * (bf16).  workspace: device memory of at least attn_bwd_workspace_bytes()
 * bytes, 256-byte aligned, owned by the caller; its contents on entry do not
 * matter and are overwritten.  Outputs must not alias inputs.
 *
 * D = 64 and 128 use the atomic-free form with seven products per tile pair
 * (FlashAttention (Metal Port) README, Documentation section): a
 * column-parallel kernel computes dK and dV, a row-parallel kernel computes
 * dQ, every gradient element is summed in one fixed order and the results
 * are bitwise reproducible.  At D = 128 a workspace of
 * attn_bwd_workspace_bytes_ds() bytes replaces the row-parallel recomputation
 * by stored dS tiles (five products per tile pair, still in a fixed order).
 * D = 256 uses the five-product form with dQ partial sums added into the
 * fp32 workspace.
 */
ATTN_API attn_status_t attn_bwd(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v, attn_tensor_t o,
                       const float* lse, attn_tensor_t dout, attn_tensor_t dq, attn_tensor_t dk,
                       attn_tensor_t dv, int B, int Hq, int Hkv, int N, int D,
                       attn_dtype_t dtype, int causal, float scale, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * Backward of attn_fwd_window (same window convention; other arguments as
 * attn_bwd).
 */
ATTN_API attn_status_t attn_bwd_window(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v,
                                       attn_tensor_t o, const float* lse, attn_tensor_t dout,
                                       attn_tensor_t dq, attn_tensor_t dk, attn_tensor_t dv,
                                       int B, int Hq, int Hkv, int N, int D,
                                       attn_dtype_t dtype, int window_left, int window_right,
                                       float scale, void* workspace, size_t workspace_bytes,
                                       void* stream);

/*
 * Backward of attn_fwd_masked: the same window and block_mask (see there);
 * other arguments as attn_bwd.  Rows that saw no key pass no gradient.  With
 * a mask: D in {64, 128} and T <= 512, else ATTN_ERR_UNSUPPORTED.
 */
ATTN_API attn_status_t attn_bwd_masked(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v,
                                       attn_tensor_t o, const float* lse, attn_tensor_t dout,
                                       attn_tensor_t dq, attn_tensor_t dk, attn_tensor_t dv,
                                       int B, int Hq, int Hkv, int N, int D,
                                       attn_dtype_t dtype, int window_left, int window_right,
                                       const uint8_t* block_mask, float scale, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * attn_bwd for callers that cannot allocate device memory.
 *
 * Some callers must not allocate GPU memory once they are running: a service
 * that reserves all of its device memory up front and forbids any later
 * cudaMalloc, or a host framework whose own allocator this library cannot
 * reach.  They cannot provide attn_bwd's workspace, so this entry point uses
 * a fixed scratch array that is part of the library itself (a static device
 * array of 64 MiB = 67108864 bytes; every GPU on which the library is loaded
 * holds it until the process exits).  It calls no cudaMalloc, cudaFree or
 * other allocating routine.  (This entry point has no counterpart in the
 * method's description; it only changes where the backward's scratch lives.)
 *
 * Arguments and results are those of attn_bwd without the workspace.  Sizes
 * whose workspace (attn_bwd_workspace_bytes) exceeds 64 MiB are rejected with
 * ATTN_ERR_WORKSPACE before anything is launched.  The first call on each
 * device looks up the scratch array's device address with that device
 * current; make that first call before any stream capture.  Every call
 * shares the one array: the kernels re-initialise everything they read from
 * it (the row statistics are rewritten and, for D = 256, the dQ accumulator
 * is zeroed on every call), but two calls whose work overlaps on the GPU (different streams, or
 * different host threads) race on it and must be serialised by the caller.
 */
ATTN_API attn_status_t attn_bwd_noalloc(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v,
                                        attn_tensor_t o, const float* lse, attn_tensor_t dout,
                                        attn_tensor_t dq, attn_tensor_t dk, attn_tensor_t dv,
                                        int B, int Hq, int Hkv, int N, int D,
                                        attn_dtype_t dtype, int causal, float scale,
                                        void* stream);

/*
 * FP8 forward (FlashAttention entity page: FP8 inference in the FlashPrefill V2
 * finding; r/mlscaling FA3 item): q, k, v are e4m3 [B, H, N, 128] tensors
 * (1-byte elements, strides in elements, 16-byte multiples) holding x / scale
 * for per-tensor scales q_scale, k_scale, v_scale; the result is attention of
 * the dequantised inputs (q_scale * q, ...) with the given softmax scale and
 * window (as attn_fwd_window): o [B, Hq, N, 128] bf16 and lse as attn_fwd.
 * Both products run on e4m3 tensor-core operands (kind::f8f6f4).  P (times
 * 32, with P <= 8 by the rescale rule) enters P V as two e4m3 terms, its
 * rounding and the rounding's residual, so it keeps about 8 significant bits (a single e4m3 term keeps 4, which
 * puts the output's error near 5 % on random inputs).  D = 128 only (else
 * ATTN_ERR_UNSUPPORTED).
 */
ATTN_API attn_status_t attn_fwd_fp8(attn_tensor_t q, attn_tensor_t k, attn_tensor_t v,
                                    attn_tensor_t o, float* lse, int B, int Hq, int Hkv, int N,
                                    int D, float q_scale, float k_scale, float v_scale,
                                    int window_left, int window_right, float scale, void* stream);

/*
 * Decode against a paged key/value cache (FlashAttention entity page:
 * FlashPrefill V2 and vLLM findings, paged KV cache and continuous batching;
 * the split-KV / decode step with a logsumexp merge).
 *
 * q [B, Hq, Sq, D] holds the Sq newest tokens of each of B sequences; query
 * token i of sequence b sits at position seqlens[b] - Sq + i.  The keys and
 * values live in 128-row pages: k_pool and v_pool describe [P, 128, Hkv, D]
 * pools (num_pages = P) with .sb = page stride, .sh = head stride, .sn = row
 * stride (elements; unit stride on D; 16-byte multiples).  Key t of sequence
 * b is row t % 128 of page block_table[b * max_pages + t / 128] (int32 device
 * array [B][max_pages]); seqlens is an int32 device array [B] with
 * 0 <= seqlens[b] <= 128 * max_pages (a length outside that range is clamped
 * into it: the sequence is taken to hold min(max(seqlens[b], 0),
 * 128 * max_pages) tokens, for its keys and its query positions alike;
 * there is no error, since the lengths are device data the host does not
 * read).  causal != 0: token i sees keys at
 * positions <= its own; otherwise all seqlens[b] keys.  Writes o [B, Hq, Sq,
 * D] (bf16) and lse [B, Hq, Sq] (fp32, natural log, contiguous); a token that
 * sees no key gets o = 0, lse = -inf.
 *
 * The page range of each (sequence, key/value head) is split so that the GPU
 * gets about four CTAs per SM; each split's partial result goes to the
 * workspace (attn_decode_workspace_bytes, 256-byte aligned, caller-owned) and
 * a second kernel merges them.  Requirements: bf16, D in {64, 128},
 * (Hq / Hkv) * Sq <= 128.  Page ids outside [0, P) read as zeros.
 */
ATTN_API size_t attn_decode_workspace_bytes(int B, int Hq, int Sq, int D, int max_pages);
ATTN_API attn_status_t attn_decode_paged(attn_tensor_t q, attn_tensor_t k_pool,
                                         attn_tensor_t v_pool, int num_pages,
                                         const int* block_table, int max_pages,
                                         const int* seqlens, attn_tensor_t o, float* lse, int B,
                                         int Hq, int Hkv, int Sq, int D, attn_dtype_t dtype,
                                         int causal, float scale, void* workspace,
                                         size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device.  Returns ATTN_OK, ATTN_ERR_DEVICE_TIMEOUT (a kernel's
 * bounded wait gave up; *where, if not NULL, receives the wait site id) or
 * ATTN_ERR_CUDA.
 */
ATTN_API attn_status_t attn_device_status(void* stream, int* where);

/*
 * Test hooks.  attn_debug_set_wait_limit_ns sets the time limit of every
 * in-kernel wait (default 2 s; 0 restores the default).
 * attn_debug_set_flags: bit 0 makes the next forward launches drop one tile
 * load, bit 1 makes the next backward launches' dK/dV kernel drop one Q tile
 * load, so that their waits run out and report ATTN_ERR_DEVICE_TIMEOUT
 * through attn_device_status (0 = normal operation).
 */
ATTN_API void attn_debug_set_wait_limit_ns(unsigned long long ns);
ATTN_API void attn_debug_set_flags(int flags);

/*
 * Choice of forward kernel for bf16 inputs with D = 128 and no block mask
 * (other forwards have one kernel each): 0 = the library's default, 1 = one
 * CTA per 128-row query tile, 2 = pairs of CTAs issuing 2-CTA tensor-core
 * products (tcgen05 .cta_group::2; FlashAttention entity page, finding
 * "FlashAttention-4: Algorithm and Kernel Pipelining for Blackwell GPUs":
 * 2-CTA MMA).  Both give the same results up to rounding order; the switch
 * exists so that the two can be compared.  Applies to calls made after it,
 * from any thread; other values select the default.
 */
ATTN_API void attn_debug_set_fwd_variant(int variant);

/*
 * Timing hook.  When both are non-NULL (cudaEvent_t handles owned by the
 * caller), the next attn_bwd call records `start` on its stream right before
 * launching its dK/dV kernel and `stop` right after it, then forgets them;
 * this times that kernel alone inside a longer stream of work.
 */
ATTN_API void attn_debug_set_bwd_events(void* start, void* stop);

/*
 * The same for the backward's row-parallel dQ kernel (head dimensions 64 and
 * 128; the D = 256 backward has no such kernel and leaves the events
 * unrecorded).
 */
ATTN_API void attn_debug_set_bwd_q_events(void* start, void* stop);

/*
 * Test hook for the exponential the softmax kernels use: y[i] = 2^x[i] for
 * n device floats, computed by the MUFU unit (mode 0) or by the FMA-pipe
 * polynomial (mode 1), asynchronously on `stream`.
 */
ATTN_API attn_status_t attn_debug_exp2(const float* x, float* y, int n, int mode, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_TILED_ATTENTION_ATTN_H_ */
