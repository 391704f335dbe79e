/*
 * libsdpa -- fused scaled-dot-product-attention forward for NVIDIA B200 (sm_100a).
 *
 * Computes, for every batch b, query head h and query row i,
 *
 *     out[b,h,i,:] = softmax_j( scale * q[b,h,i,:] . k[b,hk,j,:] + bias[i,j] + mask[b,h,i,j] ) . v[b,hk,j,:]
 *
 * (Axon PR "Add scaled_dot_product_attention", description: softmax(Q.K^T*scale
 * + mask).V over rank-4 inputs), where
 *
 *   - hk = h / (Hq / Hkv): grouped-query / multi-query attention by repeating
 *     each key/value head Hq/Hkv times consecutively (Axon PR, GQA/MQA item);
 *   - bias is the decomposed relative-position term of the SAM image encoder,
 *     computed from the UNSCALED query inside the kernel, never materialised
 *     (mlx-examples issue "segment_anything: fuse attention with
 *     mx.fast.scaled_dot_product_attention": add_decomposed_rel_pos added to
 *     (q*scale)@k^T before the softmax, and the point of fusing is not to
 *     build the T_q x T_kv matrix; candle PR "SDPA with Relative Positional
 *     Embeddings": term_h / term_w injected into the scores):
 *         bias[i,j] = q_i . Rh[qh(i) - kh(j) + Kh - 1] + q_i . Rw[qw(i) - kw(j) + Kw - 1]
 *         qh(i) = i / q_hw[1], qw(i) = i % q_hw[1], kh(j) = j / k_hw[1], kw(j) = j % k_hw[1],
 *         Kh = k_hw[0], Kw = k_hw[1] (query and key grids may differ, see sdpa_fwd);
 *   - mask is one of the Axon :mask forms (Axon PR, :mask option) -- causal
 *     with an offset, a sliding window with an offset, or a runtime additive
 *     float / boolean tensor broadcast to [B, Hq, Tq, Tkv] (mlx issue: the
 *     mask argument is an arbitrary additive array).
 *
 * Layout: every tensor is dense row-major "bhsd": q and out [B, Hq, Tq, d],
 * k and v [B, Hkv, Tkv, d], in the I/O dtype -- except for sdpa_fwd_strided,
 * which takes any batch / head / token strides (e.g. "bshd").  All data pointers are DEVICE
 * pointers owned by the caller; the library keeps no reference after a call
 * returns (it caches only TMA descriptors and a scratch buffer, see below).
 *
 * Every entry point is asynchronous on `stream` (no host synchronisation)
 * unless stated otherwise, and returns SDPA_OK (0) or a negative sdpa_status.
 * Argument errors are detected on the host before anything is launched.
 *
 * Stream order is kept as for any kernel launch.  The attention kernels are
 * launched with programmatic stream serialization and let the next grid in
 * the stream be scheduled once all their CTAs have started; each waits for
 * the grid before it (griddepcontrol.wait) before touching global memory.  A
 * caller's own kernel that follows on the same stream and is itself launched
 * with programmatic serialization must likewise wait
 * (cudaGridDependencySynchronize) before it reads this library's outputs;
 * kernels launched without that attribute need nothing.
 */
#ifndef SDPA_H_
#define SDPA_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* I/O element type.  F32 runs on the exact CUDA-core path (no TF32: the fp32
   tolerance of 1e-4 is below TF32's 10-bit mantissa); BF16 accumulates in fp32
   and rounds the output to nearest-even. */
typedef enum { SDPA_F32 = 0, SDPA_BF16 = 1 } sdpa_dtype_t;

/* Mask kinds (Axon PR, :mask option).  Readings of what the pages leave open:
   CAUSAL   key j visible from row i iff j <= i + offset.
   SLIDING  visible iff i + offset - window < j <= i + offset (window keys,
            diagonal included; one-sided, i.e. causal within the window).
   ADD_FLOAT  additive tensor in the I/O dtype (-inf allowed).
   BOOL     uint8 tensor, nonzero = attend, zero = excluded.
   A row that sees no key produces a zero output row (and lse = -inf). */
typedef enum {
  SDPA_MASK_NONE = 0,
  SDPA_MASK_CAUSAL = 1,
  SDPA_MASK_SLIDING = 2,
  SDPA_MASK_ADD_FLOAT = 3,
  SDPA_MASK_BOOL = 4
} sdpa_mask_kind_t;

/* Host-side mask description; `mask_ptr` arguments point to one of these.
   It may be NULL for NONE and for CAUSAL with offset 0.
   For ADD_FLOAT / BOOL, element (b, h, i, j) is read at
   data[b*stride_b + h*stride_h + i*stride_q + j] (element strides; a stride of
   0 broadcasts that axis; the key axis is contiguous). */
typedef struct {
  int64_t offset;     /* CAUSAL / SLIDING diagonal offset (default 0)      */
  int64_t window;     /* SLIDING window w >= 1                              */
  const void* data;   /* device pointer, ADD_FLOAT (I/O dtype) or BOOL (u8) */
  int64_t stride_b;
  int64_t stride_h;
  int64_t stride_q;
} sdpa_mask_t;

typedef enum {
  SDPA_OK = 0,
  SDPA_ERR_INVALID_ARG = -1,  /* null pointer, bad size, Hq % Hkv != 0, aliasing, ... */
  SDPA_ERR_UNSUPPORTED = -2,  /* legal request this build does not implement (d not in
                                 {16,64,128}, path forced onto a kernel that cannot
                                 take the problem) */
  SDPA_ERR_MISALIGNED = -3,   /* a pointer or stride breaks the 16-byte rule of the
                                 forced tensor-core path */
  SDPA_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed (launch, copy) */
  SDPA_ERR_TIMEOUT = -5,      /* a device-side bounded wait expired (see
                                 sdpa_last_device_error) */
  SDPA_ERR_CAPACITY = -6,     /* the request exceeds a fixed-size buffer of this entry point */
  SDPA_ERR_DEVICE_INDEX = -7  /* debug build only: a kernel's device-side index check failed
                                 (see sdpa_debug_checks) */
} sdpa_status;

/* Kernel families.  AUTO picks per shape; the others force one family and
   return SDPA_ERR_UNSUPPORTED when it cannot take the problem. */
typedef enum {
  SDPA_PATH_AUTO = 0,
  SDPA_PATH_EXACT = 1,     /* CUDA-core FFMA online softmax; every feature, fp32 and bf16 */
  SDPA_PATH_TCGEN05 = 2,   /* TMA + tcgen05/TMEM flash kernel; bf16, d in {64,128} */
  SDPA_PATH_SMALL_D = 3,   /* packed d=16 kernel, one query row per thread; bf16 */
  SDPA_PATH_SPLIT_KV = 4,  /* split-KV with in-kernel merge, short Tq / long Tkv; bf16, d=16;
                              tensor-core parts.  AUTO takes it when Tkv >= 1024 and
                              Tq <= Tkv / 16 */
  SDPA_PATH_TC_PERSISTENT = 5 /* the tcgen05 kernel as one persistent CTA per SM walking many
                                 short problems (e.g. SAM's windowed attention: 14x14-token
                                 windows); bf16, d=64, no mask, rel-pos key-grid width 14 or 16
                                 and height <= 16 or no rel-pos.  AUTO takes it from two
                                 256-row query blocks per SM and at most four key tiles each. */
} sdpa_path_t;

/*
 * sdpa_fwd -- the fused forward.
 *   q, k, v, out : device pointers (layout above).  out must not overlap q, k
 *                  or v.  k and v may be NULL only when Tkv == 0; q and out
 *                  only when B*Hq*Tq == 0.
 *   dtype        : sdpa_dtype_t of q, k, v, out, the rel-pos tables and an
 *                  ADD_FLOAT mask.
 *   B, Hq, Hkv, Tq, Tkv : B >= 0, Hq >= 1, Hkv >= 1, Hq % Hkv == 0,
 *                  Tq >= 0, Tkv >= 0.
 *   d            : head_dim, one of 16, 64, 128.
 *   scale        : score scale, finite (the Axon default 1/sqrt(d) is applied
 *                  by the Python binding, not here).
 *   mask_kind, mask_ptr : sdpa_mask_kind_t and a host sdpa_mask_t* (see above).
 *   rel_pos_h, rel_pos_w : device tables [q_hw[0]+k_hw[0]-1, d] and
 *                  [q_hw[1]+k_hw[1]-1, d] (2*K-1 rows each when the grids are
 *                  equal) in the I/O dtype, shared by every batch and head;
 *                  both NULL disables the bias, exactly one NULL is INVALID_ARG.
 *   q_hw, k_hw   : host int[2] patch grids (height, width) with
 *                  q_hw[0]*q_hw[1] == Tq and k_hw[0]*k_hw[1] == Tkv; required
 *                  with rel-pos, ignored otherwise.  The grids may differ:
 *                  the bias formula above is read with qh, qw from the query
 *                  grid and kh, kw and the shifts Kh-1, Kw-1 from the key
 *                  grid, so table row qh-kh+Kh-1 covers offsets -(Kh-1) ..
 *                  Qh-1 (no interpolation of resized tables).
 *   stream       : CUDA stream the work is enqueued on.
 */
int sdpa_fwd(const void* q, const void* k, const void* v, void* out, sdpa_dtype_t dtype,
             int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale,
             int mask_kind, const void* mask_ptr,
             const void* rel_pos_h, const void* rel_pos_w,
             const int* q_hw, const int* k_hw,
             cudaStream_t stream);

/*
 * sdpa_fwd_ex -- sdpa_fwd plus two options.
 *   lse  : NULL, or a device float [B, Hq, Tq] receiving the natural-log
 *          sum-exp of each score row (m + log l; -inf for a row with no
 *          visible key).
 *   path : sdpa_path_t; AUTO behaves like sdpa_fwd.  A forced family that
 *          cannot take the problem returns SDPA_ERR_UNSUPPORTED (or
 *          SDPA_ERR_MISALIGNED) before any device work.
 * The persistent tensor-core path allocates nothing and writes no scratch.
 * The split-KV path merges its parts inside a thread-block cluster when the
 * key axis fits in 8 parts of 512 keys and there are at most 64 query rows;
 * otherwise -- and the tensor-core path when it splits a key range -- it
 * keeps partial results in a scratch buffer that the library allocates on
 * first use per device and grows when needed (never freed until exit); calls
 * on one device that overlap on the GPU must not use such a path concurrently.
 * Growing that buffer is the one place an otherwise asynchronous call blocks
 * the host: before it frees the smaller buffer it calls
 * cudaDeviceSynchronize(), because earlier launches may still be using it.
 * A caller that wants no such stall makes one call at its largest size first.
 * lse must not overlap q, k, v, out or the mask tensor (SDPA_ERR_INVALID_ARG).
 */
int sdpa_fwd_ex(const void* q, const void* k, const void* v, void* out, sdpa_dtype_t dtype,
                int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale,
                int mask_kind, const void* mask_ptr,
                const void* rel_pos_h, const void* rel_pos_w,
                const int* q_hw, const int* k_hw,
                float* lse, int path, cudaStream_t stream);

/*
 * sdpa_fwd_strided -- sdpa_fwd_ex on tensors with arbitrary batch, head and
 * token strides, e.g. the "bshd" layout [B, T, H, d] that the Axon PR ("Add
 * scaled_dot_product_attention", :axes option) takes by default, used in
 * place (the PR's review asks to avoid the transposes to "bhsd").
 *
 * Each sdpa_strides_t holds the ELEMENT strides of the batch, head and token
 * axes of one tensor; the head_dim axis is contiguous.  A NULL strides pointer
 * means dense bhsd for that tensor: q and out {Hq*Tq*d, Tq*d, d}, k and v
 * {Hkv*Tkv*d, Tkv*d, d}; bshd is {T*H*d, d, H*d}.  Strides must be positive
 * (SDPA_ERR_INVALID_ARG otherwise).  The tensor-core path and the head_dim-16
 * paths also need every stride to be a multiple of 8 elements for bf16 (their
 * 16-byte TMA boxes and row loads); AUTO sends other problems to the exact
 * kernel, an explicit path returns SDPA_ERR_MISALIGNED.  `out` must not
 * overlap any input over their address spans (SDPA_ERR_INVALID_ARG).  lse,
 * when given, is dense [B, Hq, Tq] as for sdpa_fwd_ex.
 */
typedef struct {
  int64_t b;  /* batch stride (elements) */
  int64_t h;  /* head stride  (elements) */
  int64_t t;  /* token stride (elements) */
} sdpa_strides_t;

int sdpa_fwd_strided(const void* q, const sdpa_strides_t* q_strides,
                     const void* k, const sdpa_strides_t* k_strides,
                     const void* v, const sdpa_strides_t* v_strides,
                     void* out, const sdpa_strides_t* out_strides,
                     sdpa_dtype_t dtype, int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale,
                     int mask_kind, const void* mask_ptr,
                     const void* rel_pos_h, const void* rel_pos_w,
                     const int* q_hw, const int* k_hw,
                     float* lse, int path, cudaStream_t stream);

/*
 * sdpa_merge -- combine attention results over disjoint key subsets of the
 * same queries into the result over their union, e.g. a long key axis run
 * chunk by chunk through sdpa_fwd_ex with its lse output.  Part i gives
 * out_i [B, Hq, Tq, d] (I/O dtype, dense bhsd) and lse_i [B, Hq, Tq] (float,
 * natural-log sum-exp of its score rows, -inf where it saw no key).  Writes
 *     lse = L = log sum_i exp(lse_i),   out = sum_i exp(lse_i - L) * out_i
 * -- the softmax numerators of every key summed, as attention over the whole
 * key axis does (Axon PR "Add scaled_dot_product_attention": softmax(Q.K^T *
 * scale + mask).V).  A row whose parts are all -inf gets zeros and -inf.
 *   outs, lses : HOST arrays of `nparts` DEVICE pointers, 1 <= nparts <= 16.
 *   out        : device output; may be outs[0] (in place), must not overlap
 *                any other part.  16-byte aligned, as must every outs[i].
 *   lse        : device float output or NULL; may be lses[0].
 * d must be 16, 64 or 128.  Errors: SDPA_ERR_INVALID_ARG (counts, NULLs,
 * overlap), SDPA_ERR_UNSUPPORTED (d), SDPA_ERR_MISALIGNED.  Asynchronous on
 * `stream`.
 */
int sdpa_merge(const void* const* outs, const float* const* lses, int nparts,
               void* out, float* lse, sdpa_dtype_t dtype, int B, int Hq, int Tq, int d,
               cudaStream_t stream);

/* The path AUTO would take for this problem (a non-negative sdpa_path_t), or a
   negative sdpa_status when the arguments are invalid.  Launches nothing;
   pointers are only checked for NULL and alignment. */
int sdpa_select_path(const void* q, const void* k, const void* v, void* out, sdpa_dtype_t dtype,
                     int B, int Hq, int Hkv, int Tq, int Tkv, int d,
                     int mask_kind, const void* mask_ptr,
                     const void* rel_pos_h, const void* rel_pos_w,
                     const int* q_hw, const int* k_hw);

/*
 * sdpa_fwd_host -- the same forward on HOST buffers.  Copies q, k, v, the
 * rel-pos tables and an ADD_FLOAT/BOOL mask (its data pointer is then a HOST
 * pointer, read with the strides given) to device buffers the library keeps
 * per device (grown as needed), runs sdpa_fwd_ex on `stream`, copies the
 * result into the host buffer `out` and synchronises `stream` before
 * returning.  For transfer speed the host buffers should be pinned.  Not
 * reentrant across host threads on the same device.
 */
int sdpa_fwd_host(const void* q, const void* k, const void* v, void* out, sdpa_dtype_t dtype,
                  int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale,
                  int mask_kind, const void* mask_ptr,
                  const void* rel_pos_h, const void* rel_pos_w,
                  const int* q_hw, const int* k_hw,
                  int path, cudaStream_t stream);

/*
 * sdpa_fwd_split_kv_static -- the split-KV forward (bf16, head_dim 16, every
 * mask kind, no rel-pos) for callers that cannot allocate device memory during
 * a call, e.g. code running under a memory pool it does not own or whose
 * start-up already reserved all the memory it may use.  (The pages have no
 * counterpart; this is an entry point of the library, not of the method.)
 *
 * It allocates nothing: its scratch is a fixed 4 MiB device array inside the
 * library (64 KiB of tickets, one per (batch, head), and the partial results),
 * held by every device that loads the library until the process exits.
 * Problems whose scratch does not fit return SDPA_ERR_CAPACITY; an
 * unsupported shape returns SDPA_ERR_UNSUPPORTED.  q, k, v, out (and lse, may
 * be NULL) are caller-owned device pointers exactly as for sdpa_fwd_ex.
 *
 * The first call on a device looks up the array's device address; make that
 * first call before capturing a stream into a graph.  Every call on a device
 * shares the array and leaves its contents behind: calls whose kernels may
 * overlap on the GPU (different streams without ordering between them) race
 * on it and must not be issued; calls on one stream are ordered and safe.
 * Such a race is not detected: it gives wrong output silently, not an error
 * status from sdpa_last_device_error.
 */
int sdpa_fwd_split_kv_static(const void* q, const void* k, const void* v, void* out, sdpa_dtype_t dtype,
                             int B, int Hq, int Hkv, int Tq, int Tkv, int d, float scale,
                             int mask_kind, const void* mask_ptr, float* lse, cudaStream_t stream);

/* Synchronises `stream`, then returns and clears the device error word of the
   current device: SDPA_OK; SDPA_ERR_DEVICE_INDEX when, in a debug build, a
   kernel's index check failed since the last call; SDPA_ERR_TIMEOUT when a
   kernel gave up a bounded wait since the last call (output undefined in
   either case); or SDPA_ERR_CUDA when the synchronisation itself failed. */
int sdpa_last_device_error(cudaStream_t stream);

/* 1 when this library was built with SDPA_DEBUG (libsdpa_debug.so), else 0.
   A debug build tests every index its kernels derive -- query and key rows,
   rel-pos table rows (the qh - kh + Kh - 1 and qw - kw + Kw - 1 of the
   decomposed bias), mask and workspace slots, shared-memory slots of the
   rel-pos scatter -- against its extent before the access.  A failed check
   skips the access and sets the device error word, which
   sdpa_last_device_error reports as SDPA_ERR_DEVICE_INDEX: no trap, fault or
   hang.  Results of a debug build equal the release build's; only speed
   differs.  Host-only: needs no GPU. */
int sdpa_debug_checks(void);

/* Self-test of the device-side index checks (the library's own
   instrumentation; the pages have no counterpart).  Enqueues on `stream` one
   kernel whose single thread evaluates the index check of `index` against
   [0, extent) and touches no memory at `index`.  In a debug build an index
   outside the extent sets the device error word (the next
   sdpa_last_device_error returns SDPA_ERR_DEVICE_INDEX); in a release build
   the check is compiled out and nothing is set.  extent < 0:
   SDPA_ERR_INVALID_ARG before any launch. */
int sdpa_selftest_index_check(long long index, long long extent, cudaStream_t stream);

/* Self-test of the failure detection above (the pages have no counterpart;
   it checks this library's own error path).  Enqueues on `stream` one kernel
   whose single thread waits, bounded by limit_ns nanoseconds of %globaltimer,
   on an mbarrier that nothing arrives on -- the same bounded wait every
   tensor-core kernel uses -- and so sets the device error word exactly as an
   expired wait inside a forward call would.  The next sdpa_last_device_error
   then returns SDPA_ERR_TIMEOUT and clears the word.  No fault, trap or hang
   is involved and the CUDA context stays usable.  limit_ns must be in
   (0, 2e9]: SDPA_ERR_INVALID_ARG otherwise, before any launch. */
int sdpa_selftest_wait_timeout(unsigned long long limit_ns, cudaStream_t stream);

/* Static description of a status code (never NULL). */
const char* sdpa_strerror(int status);

/* Library version, major*10000 + minor*100 + patch. */
int sdpa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SDPA_H_ */
