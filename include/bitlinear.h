/*
 * bitlinear.h - C ABI of libbitlinear, the B200 (sm_100a) BitNet b1.58
 * BitLinear (W1.58-A8) hot path:  y = F.linear(ActQuant(x), WeightQuant(W)).
 *
 * Definitions followed (page title, section):
 *   WeightQuant  "Core AI model zoo - BitVLA", section 1: per-tensor absmean,
 *                s = 1/mean(|W|), code = round(W*s).clamp(-1, 1); also
 *                "BitNet-Embeddings I2_S guide", section 3.3 (I2_S packing).
 *   ActQuant     BitVLA page, section 1: per-token int8 absmax,
 *                q = round(x*127/max|x|).clamp(-128, 127).
 *   Storage      BitVLA page, section 2: codes stored as code+1, 16 codes per
 *                32-bit word, K only needs K % 16 == 0, N need not be a
 *                multiple of 32, and the scale D is one fp32 per output row,
 *                laid out [N, 1].
 *   Product      BitVLA page, section 2: the wrapper applies ActQuant before
 *                the kernel, so the result equals
 *                F.linear(ActQuant(x), WeightQuant(W)).
 *
 * Numerics (identical to the CPU oracle, bit for bit):
 *   mean  = mean(|W|) over the whole tensor, exact sum, correctly rounded
 *           to fp32; mean_c = max(mean, 1e-5);  s = RN(1 / mean_c)
 *   code  = clamp(rint(RN(W * s)), -1, 1)      (rint: half to even)
 *   packed word n*(K/16) + k/16, bits [2*(k%16), 2*(k%16)+2) = code + 1
 *   D[n]  = mean_c for every row n
 *   s_x   = RN(127 / max(max_k |x[m,k]|, 1e-5))
 *   q     = clamp(rint(RN(x * s_x)), -128, 127)
 *   acc   = sum_k q[m,k] * code[n,k]          (exact int32)
 *   y     = RN( RN(float(acc) / s_x[m]) * D[n] )
 *
 * Conventions for every entry point:
 *   - All pointers named "device" are device pointers on the current CUDA
 *     device; the caller owns every buffer. This library allocates nothing and
 *     keeps no state beyond cached device attributes, with one exception: the
 *     fixed scratch array of bitlinear_forward_noalloc (16 MiB in the device
 *     image of every GPU that loads the library) and its cached device
 *     address per GPU.
 *   - Matrices are dense row-major with no padding: x [M,K] fp32, W [N,K] fp32,
 *     packed [N, K/16] uint32, D [N] fp32 (a torch [N,1] tensor), y [M,N] fp32.
 *   - Device buffers must be 16-byte aligned, the workspace 256-byte aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). Entry points marked "synchronous" synchronise that stream.
 *   - No exception crosses this boundary and no kernel traps; every error is a
 *     returned bl_status. Kernels that wait on barriers give up after a bounded
 *     time and record the failure in the workspace (see
 *     bitlinear_workspace_error).
 *   - Limits: 0 < K <= 131072 and K % 16 == 0 (so |acc| < 2^24 and fp32
 *     holds it exactly); 0 <= M, N <= 2^31 - 1. M == 0 or N == 0 is a no-op.
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BL_API __attribute__((visibility("default")))
#else
#define BL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* bl_stream_t;

typedef enum {
  BL_OK = 0,
  BL_ERR_NULL = 1,        /* a required pointer is NULL */
  BL_ERR_SHAPE = 2,       /* K % 16 != 0, K <= 0, K > 131072, or M/N out of range */
  BL_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned (workspace: 256) */
  BL_ERR_WORKSPACE = 4,   /* ws_bytes smaller than the *_workspace_size query */
  BL_ERR_NONFINITE = 5,   /* pack: W holds Inf or NaN, so mean(|W|) is not finite */
  BL_ERR_DEVICE = 6,      /* a kernel recorded a device-side failure (bounded wait expired) */
  BL_ERR_CUDA = 7,        /* a CUDA runtime call failed (launch, copy, attribute) */
  BL_ERR_UNSUPPORTED = 8, /* the current device is not sm_100 (B200 class) */
  BL_ERR_FORMAT = 9       /* I2_S: a field holds 3, the scale is not finite and
                             positive, or (export) the rows of D differ */
} bl_status;

/* Version of this ABI (incremented on any incompatible change). */
BL_API int bitlinear_abi_version(void);

/* Static string identifying the sources this library was built from (a hash
 * of the kernel sources and this header, set by the build); never NULL. */
BL_API const char* bitlinear_build_id(void);

/* Static string for a status code; never NULL. */
BL_API const char* bitlinear_status_string(int status);

/* BL_OK if the current device can run the kernels (compute capability 10.0). */
BL_API int bitlinear_device_check(void);

/* ---------------------------------------------------------------- pack --- */

/* Bytes of scratch that bitlinear_pack_weights needs (a few KB). */
BL_API size_t bitlinear_pack_workspace_size(int64_t N, int64_t K);

/* WeightQuant + 2-bit pack (BitVLA page sections 1 and 2; I2_S guide 3.3).
 *   W       device fp32 [N, K], read only.
 *   packed  device uint32 [N, K/16], fully overwritten.
 *   D       device fp32 [N] (the [N,1] scale), every entry set to mean_c.
 *   ws      device scratch of ws_bytes >= bitlinear_pack_workspace_size().
 * Synchronous: it waits on `stream` so that it can report BL_ERR_NONFINITE
 * (packed and D are left unwritten in that case). N >= 1 is required. */
BL_API int bitlinear_pack_weights(const float* W, int64_t N, int64_t K,
                           uint32_t* packed, float* D,
                           void* ws, size_t ws_bytes, bl_stream_t stream);

/* As bitlinear_pack_weights, from a bf16 master weight: W holds the bf16 bit
 * patterns [N, K] (uint16, 16-byte aligned). Each value is widened to fp32
 * exactly (a bf16 is the upper half of an fp32), then quantised as above
 * ("Core AI model zoo - BitVLA" section 1: the checkpoint is a bf16 latent
 * master, quantised on the fly). Synchronous. */
BL_API int bitlinear_pack_weights_bf16(const uint16_t* W, int64_t N, int64_t K,
                                       uint32_t* packed, float* D,
                                       void* ws, size_t ws_bytes, bl_stream_t stream);

/* As bitlinear_pack_weights, without synchronising: the pack is enqueued on
 * `stream` and a non-finite weight is OR-ed into the status word at the start
 * of `ws` instead of being returned (that call then writes neither packed nor
 * D; later calls are not affected). The caller zeroes that word before the
 * first call (a zero-filled workspace); bitlinear_pack_status reads it.
 * Calls that share `ws` must be ordered on one stream. */
BL_API int bitlinear_pack_weights_async(const float* W, int64_t N, int64_t K,
                                        uint32_t* packed, float* D,
                                        void* ws, size_t ws_bytes, bl_stream_t stream);

/* Synchronises `stream`, reads and clears the status word of a pack
 * workspace: BL_OK if no asynchronous pack since the last read met a
 * non-finite weight, else BL_ERR_NONFINITE. */
BL_API int bitlinear_pack_status(void* ws, size_t ws_bytes, bl_stream_t stream);

/* ------------------------------------------------------------ ActQuant --- */

/* Per-token int8 absmax quantisation (BitVLA page section 1).
 *   x       device fp32 [M, K].
 *   q       device int8 [M, K], natural column order.
 *   s_x     device fp32 [M]: the scale 127/max|x| (not its reciprocal).
 *   rowsum  device int32 [M] or NULL: sum_k q[m,k] (exact).
 * Asynchronous. */
BL_API int bitlinear_quant_act(const float* x, int64_t M, int64_t K,
                        int8_t* q, float* s_x, int32_t* rowsum,
                        bl_stream_t stream);

/* As bitlinear_quant_act, from bf16 activations (uint16 bit patterns [M, K],
 * widened to fp32 exactly). Asynchronous. */
BL_API int bitlinear_quant_act_bf16(const uint16_t* x, int64_t M, int64_t K,
                                    int8_t* q, float* s_x, int32_t* rowsum, bl_stream_t stream);

/* ------------------------------------------------------------- forward --- */

/* Bytes of scratch that bitlinear_forward / bitlinear_forward_acc need:
 * the quantised activations (M*K bytes, in a kernel-private column order),
 * s_x and row sums (4*M bytes each) and a 256-byte header holding the
 * device error word. */
BL_API size_t bitlinear_workspace_size(int64_t M, int64_t N, int64_t K);

/* y = F.linear(ActQuant(x), WeightQuant(W)) from packed weights (BitVLA page
 * section 2: the wrapper applies ActQuant, then the ternary kernel).
 *   x       device fp32 [M, K].
 *   packed  device uint32 [N, K/16] from bitlinear_pack_weights.
 *   D       device fp32 [N] per-row scale.
 *   y       device fp32 [M, N], fully overwritten; nothing outside it is written.
 *   ws      device scratch, ws_bytes >= bitlinear_workspace_size(M, N, K).
 * M <= 16 runs the decode kernel: every CTA quantises x itself and the packed
 * weights stream once through a shared-memory ring (K up to about 13000 for
 * M <= 8; wider rows take the tensor-core path). Larger M quantises into ws
 * and runs the tcgen05 tensor-core GEMM. Asynchronous. */
BL_API int bitlinear_forward(const float* x, int64_t M, int64_t N, int64_t K,
                      const uint32_t* packed, const float* D, float* y,
                      void* ws, size_t ws_bytes, bl_stream_t stream);

/* As bitlinear_forward, from bf16 activations: x holds bf16 bit patterns
 * [M, K] (uint16, 16-byte aligned), widened to fp32 exactly inside the
 * quantiser; y is fp32 [M, N]. Same workspace. Asynchronous. */
BL_API int bitlinear_forward_bf16(const uint16_t* x, int64_t M, int64_t N, int64_t K,
                                  const uint32_t* packed, const float* D, float* y,
                                  void* ws, size_t ws_bytes, bl_stream_t stream);

/* As bitlinear_forward, but writes the exact int32 accumulators
 * acc[m,n] = sum_k q[m,k] * code[n,k] to device int32 [M, N] instead of y. */
BL_API int bitlinear_forward_acc(const float* x, int64_t M, int64_t N, int64_t K,
                          const uint32_t* packed, int32_t* acc,
                          void* ws, size_t ws_bytes, bl_stream_t stream);

/* Two-phase form of bitlinear_forward for projections that share one input
 * (q/k/v, or gate/up): quantise x once, then contract with several weights.
 * bitlinear_prepare_act writes the int8 codes (kernel-private column order),
 * s_x and row sums of x [M,K] into ws (ws_bytes >=
 * bitlinear_workspace_size(M, N, K) for any N). Asynchronous. */
BL_API int bitlinear_prepare_act(const float* x, int64_t M, int64_t K,
                                 void* ws, size_t ws_bytes, bl_stream_t stream);

/* Contraction + rescale from a workspace filled by bitlinear_prepare_act with
 * the same M and K: y [M,N] = RN(RN(acc/s_x) * D). Runs the decode kernel
 * (prepared codes copied into shared memory) for M <= 16 and the tcgen05
 * tensor-core kernel otherwise. The workspace is only read (and its error
 * word reset), so several calls may follow one prepare. Asynchronous. */
BL_API int bitlinear_forward_prepared(int64_t M, int64_t N, int64_t K,
                                      const uint32_t* packed, const float* D, float* y,
                                      void* ws, size_t ws_bytes, bl_stream_t stream);

/* Forward from pre-quantised activations: q device int8 [M, K] in natural
 * column order and s_x device fp32 [M] (the scale 127/max|x| per token), as
 * bitlinear_quant_act writes them. y [M,N] = RN(RN(acc/s_x) * D) with
 * acc = sum_k q*code exactly. Any int8 codes are accepted (-128 included).
 * q, packed, D and y must be 16-byte aligned, ws 256-byte aligned with
 * ws_bytes >= bitlinear_workspace_size(M, N, K). Reorders q into ws, then runs
 * the contraction of bitlinear_forward_prepared. Asynchronous. */
BL_API int bitlinear_forward_q(const int8_t* q, const float* s_x, int64_t M, int64_t N, int64_t K,
                               const uint32_t* packed, const float* D, float* y,
                               void* ws, size_t ws_bytes, bl_stream_t stream);

/* Per-projection RMSNorm then ActQuant ("BitNet-Embeddings I2_S guide"
 * section 3.1: x -> RMSNorm(x, norm.weight) -> activation_quant -> matmul;
 * rms_norm_eps 1e-6). Per token: ms = mean(x^2), the exact mean correctly
 * rounded to fp32 once; r = RN(1/RN(sqrt(RN(ms + eps)))); n = RN(RN(x*r)*g);
 * then the ActQuant of bitlinear_quant_act on n (q, s_x, rowsum as there).
 *   x  device fp32 [M, K]; g device fp32 [K] (the projection's norm.weight);
 *   eps >= 0 (finite). K <= 16384; x, g, q 16-byte aligned. Asynchronous. */
BL_API int bitlinear_rmsnorm_quant_act(const float* x, const float* g, float eps, int64_t M, int64_t K,
                                       int8_t* q, float* s_x, int32_t* rowsum, bl_stream_t stream);

/* y = F.linear(ActQuant(RMSNorm(x, g)), WeightQuant(W)) from packed weights.
 * M <= 16: one decode-kernel launch whose CTAs normalise and quantise x
 * themselves. Larger M: the fused norm + quantiser writes the codes into ws,
 * then the tensor-core kernel runs. Same arguments as bitlinear_forward plus g
 * and eps; K <= 16384. Asynchronous. */
BL_API int bitlinear_forward_rmsnorm(const float* x, const float* g, float eps, int64_t M, int64_t N,
                                     int64_t K, const uint32_t* packed, const float* D, float* y,
                                     void* ws, size_t ws_bytes, bl_stream_t stream);

/* ------------------------------------------- per-256-block scale variant --- */

/* "Core AI model zoo - BitVLA" section 2 contrasts BitNet's per-row scale
 * D [N, 1] with BitCPM's per-256-block scale, which it names without defining.
 * Reading implemented here: a block is 256 consecutive columns of one row
 * (the last block of a row holds K % 256 columns when that is not zero); each
 * block is quantised with the per-tensor formula above applied to the block
 * alone (exact mean of |W| over the block, floor 1e-5, s = RN(1/mean_c),
 * code = clamp(rint(RN(W*s)), -1, 1)); the packed words are the same format;
 * D is fp32 [N, nb] row-major with nb = ceil(K / 256), D[n,b] = mean_c of
 * block (n, b). The product, per token m and row n:
 *   acc_b = sum over block b's columns of q[m,k] * code[n,k]   (exact)
 *   t_b   = RN( RN(float(acc_b) / s_x[m]) * D[n,b] )
 *   y     = t_0, then y = RN(y + t_b) for b = 1 .. nb-1 (ascending order). */

/* nb = ceil(K / 256), the number of scale blocks per row; 0 for an invalid K. */
BL_API int64_t bitlinear_block_scales(int64_t K);

/* WeightQuant per 256-column block + 2-bit pack.
 *   W       device fp32 [N, K], read only.
 *   packed  device uint32 [N, K/16], fully overwritten.
 *   D       device fp32 [N, nb], fully overwritten.
 *   ws      device scratch of ws_bytes >= bitlinear_pack_workspace_size().
 * Synchronous (it reads back the status word). BL_ERR_NONFINITE if a block
 * holds Inf or NaN; that block's words and scale are then left unwritten and
 * every other block is packed. N >= 1 is required. */
BL_API int bitlinear_pack_weights_blocks(const float* W, int64_t N, int64_t K,
                                         uint32_t* packed, float* D,
                                         void* ws, size_t ws_bytes, bl_stream_t stream);

/* As bitlinear_pack_weights_blocks, from a bf16 master weight (bit patterns
 * [N, K], uint16, 16-byte aligned), each value widened to fp32 exactly.
 * Synchronous. */
BL_API int bitlinear_pack_weights_blocks_bf16(const uint16_t* W, int64_t N, int64_t K,
                                              uint32_t* packed, float* D,
                                              void* ws, size_t ws_bytes, bl_stream_t stream);

/* Bytes of scratch that bitlinear_forward_blocks needs: the forward
 * workspace plus one int32 per token and block (the row sums of the codes per
 * block, for the tensor-core route). */
BL_API size_t bitlinear_blocks_workspace_size(int64_t M, int64_t N, int64_t K);

/* y [M, N] from per-block scaled weights (packed and D from
 * bitlinear_pack_weights_blocks). One token with K % 256 == 0 and K <= 8192:
 * one launch that quantises x in every CTA. M < 128: ActQuant into ws, then a
 * CUDA-core kernel that contracts each 256-column block with dp4a and adds the
 * block terms in ascending order. M >= 128: ActQuant into ws, the codes' row
 * sums per block, then one tcgen05 tensor-core GEMM per block over its 256
 * columns whose epilogue applies that block's D and adds the term to y (the
 * first block stores it). ws_bytes >= bitlinear_blocks_workspace_size(M, N,
 * K); every device pointer 16-byte aligned, ws 256-byte aligned.
 * Asynchronous. */
BL_API int bitlinear_forward_blocks(const float* x, int64_t M, int64_t N, int64_t K,
                                    const uint32_t* packed, const float* D, float* y,
                                    void* ws, size_t ws_bytes, bl_stream_t stream);

/* As bitlinear_forward_blocks, from bf16 activations (bit patterns [M, K],
 * uint16, 16-byte aligned), widened to fp32 exactly in the quantiser; y fp32.
 * Same workspace. Asynchronous. */
BL_API int bitlinear_forward_blocks_bf16(const uint16_t* x, int64_t M, int64_t N, int64_t K,
                                         const uint32_t* packed, const float* D, float* y,
                                         void* ws, size_t ws_bytes, bl_stream_t stream);

/* ---------------------------------------------------------------- batch --- */

/* One BitLinear of a batch: y [M,N] = F.linear(ActQuant(x [M,K]), W) from
 * packed [N, K/16] and D [N] (same meaning and layout as bitlinear_forward). */
typedef struct {
  const float* x;
  int64_t M;
  int64_t N;
  int64_t K;
  const uint32_t* packed;
  const float* D;
  float* y;
} bl_linear_call;

/* Flag for bitlinear_forward_batch: the packed weights and D of the calls are
 * not written by the work enqueued on `stream` just before the batch (as in a
 * decode loop, where weights are static). The decode kernels may then start
 * streaming them while that work still runs (programmatic dependent launch);
 * activations are still read only after it has finished. */
#define BL_FLAG_STREAM_WEIGHTS_EARLY 1u

/* Flag for bitlinear_forward_batch: give every call its own launch, in order
 * (for calls that stand for dependent layers; with the flag above, each
 * launch may still stream its weights while the one before it runs). Without
 * it, consecutive decode-sized calls share launches. */
#define BL_FLAG_ONE_LAUNCH_PER_CALL 2u

/* Bytes of scratch for bitlinear_forward_batch: the largest
 * bitlinear_workspace_size of its calls. */
BL_API size_t bitlinear_batch_workspace_size(const bl_linear_call* calls, int count);

/* Runs `count` independent BitLinears, in order, on `stream`. Consecutive
 * decode-sized calls (M <= 16) are fused into one launch of up to 8 calls
 * (one persistent kernel streams all of their packed weights); other calls
 * run through the tensor-core path one at a time. No output may overlap any
 * input or another output of the same batch. A one-call batch without flags
 * is the same as bitlinear_forward. Errors of any call are reported before
 * anything is launched. Asynchronous. */
BL_API int bitlinear_forward_batch(const bl_linear_call* calls, int count, uint32_t flags,
                                   void* ws, size_t ws_bytes, bl_stream_t stream);

/* Scratch for bitlinear_forward_host: the forward workspace plus room for x
 * and y on the device. */
BL_API size_t bitlinear_host_workspace_size(int64_t M, int64_t N, int64_t K);

/* End-to-end call with HOST activations: copies x_host (fp32 [M,K], pinned
 * memory recommended) to the device, runs bitlinear_forward, copies y back to
 * y_host (fp32 [M,N]) and synchronises `stream`. packed and D are device
 * buffers (the weights stay resident). Synchronous. */
BL_API int bitlinear_forward_host(const float* x_host, int64_t M, int64_t N, int64_t K,
                           const uint32_t* packed, const float* D, float* y_host,
                           void* ws, size_t ws_bytes, bl_stream_t stream);

/* The same three steps as bitlinear_forward_host, enqueued on `stream`
 * without synchronising: y_host holds the result once the stream has been
 * synchronised. x_host and y_host must be pinned (page-locked) for the copies
 * to overlap the host; they must stay valid and untouched until then. Calls on
 * one stream may share a workspace (stream order serialises them). */
BL_API int bitlinear_forward_host_async(const float* x_host, int64_t M, int64_t N, int64_t K,
                                 const uint32_t* packed, const float* D, float* y_host,
                                 void* ws, size_t ws_bytes, bl_stream_t stream);

/* Scratch for bitlinear_forward_batch_host: the batch workspace plus device
 * room for every call's x and y. */
BL_API size_t bitlinear_batch_host_workspace_size(const bl_linear_call* calls, int count);

/* bitlinear_forward_batch with HOST activations and outputs: calls[i].x and
 * calls[i].y are host pointers (pinned memory for the copies to run
 * asynchronously), packed and D device pointers. Copies every x to the device
 * (calls whose host blocks follow one another in host memory move in one
 * copy), runs the batch with `flags`, and copies every y back the same way.
 * Nothing is synchronised: the outputs are in host memory once `stream` has
 * been synchronised. Errors of any call are reported before anything runs. */
BL_API int bitlinear_forward_batch_host(const bl_linear_call* calls, int count, uint32_t flags,
                                        void* ws, size_t ws_bytes, bl_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word in a
 * forward workspace. BL_OK if no kernel recorded a failure, else
 * BL_ERR_DEVICE. */
BL_API int bitlinear_workspace_error(void* ws, size_t ws_bytes, bl_stream_t stream);

/* Size of the fixed device scratch used by bitlinear_forward_noalloc:
 * 16 MiB per GPU that loads this library, held until the process exits. */
#define BITLINEAR_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* bitlinear_forward for callers that cannot allocate device memory: a plugin
 * whose host framework owns all device memory through its own allocator, a C
 * program with no device allocator of its own, or a latency-critical loop that
 * cannot afford cudaMalloc's possible device synchronisation. The pages have no
 * counterpart; this is an interface convenience, not part of the method.
 *   x, packed, D, y   as for bitlinear_forward (the caller still owns them).
 * Scratch: instead of a caller workspace, the call uses a 16 MiB array in the
 * library's device image (BITLINEAR_NOALLOC_SCRATCH_BYTES). It returns
 * BL_ERR_WORKSPACE, without touching the GPU, when
 * bitlinear_workspace_size(M, N, K) exceeds that size (e.g. M*K above about
 * 16.7 million). It calls no cudaMalloc, cudaFree or other allocating routine.
 * The first call on a device looks up the array's device address there (once
 * per device, with that device current); make that first call before any
 * stream capture. Every call shares the one array per device, and the array
 * keeps the last call's contents. Calls that can overlap on the same GPU
 * (other streams, other host threads) race on it and must be serialised by the
 * caller. The device error word of these calls is the first word of that
 * array; bitlinear_noalloc_error reads it. Asynchronous. */
BL_API int bitlinear_forward_noalloc(const float* x, int64_t M, int64_t N, int64_t K,
                                     const uint32_t* packed, const float* D, float* y,
                                     bl_stream_t stream);

/* The device error word of bitlinear_forward_noalloc, as
 * bitlinear_workspace_error reads it for a caller workspace: synchronises
 * `stream`, then reads and clears the word at the start of the fixed scratch
 * of the current device. BL_OK if no call recorded a failure since the last
 * read, BL_ERR_DEVICE if a kernel's bounded wait expired (its y is then
 * incomplete), BL_ERR_CUDA if the scratch's address cannot be found. Allocates
 * nothing. */
BL_API int bitlinear_noalloc_error(bl_stream_t stream);

/* Diagnostic: bitlinear_selftest_wait_timeout on the fixed scratch of
 * bitlinear_forward_noalloc, so that bitlinear_noalloc_error then reports
 * BL_ERR_DEVICE. No fault, trap or hang is involved. Asynchronous. */
BL_API int bitlinear_noalloc_selftest_wait_timeout(uint64_t limit_ns, bl_stream_t stream);

/* ---------------------------------------------------------------- I2_S --- */

/* I2_S, the 2-bit ternary format of the "BitNet-Embeddings I2_S guide"
 * (section "I2_S Ternary Packing"): codes stored as code + 1 (-1 -> 0,
 * 0 -> 1, +1 -> 2), 128 values per 32-byte block with
 * byte = c0 << 6 | c1 << 4 | c2 << 2 | c3, and the fp32 scale 1/mean(|w|)
 * appended (little-endian) right after the last block. The blocks run over the
 * flattened row-major [N, K] tensor; a tail shorter than 128 values is padded
 * with the code 0. The page does not say which four values of a block share a
 * byte; `layout` picks the reading:
 *   BL_I2S_CONSECUTIVE  byte j holds values 4j, 4j+1, 4j+2, 4j+3 (c0..c3);
 *   BL_I2S_QUARTERS     byte j holds values j, j+32, j+64, j+96 (c0..c3). */
#define BL_I2S_CONSECUTIVE 0
#define BL_I2S_QUARTERS 1

/* Bytes of the I2_S buffer of an [N, K] tensor: 32 * ceil(N*K / 128) + 4
 * (0 for negative sizes). */
BL_API size_t bitlinear_i2s_bytes(int64_t N, int64_t K);

/* Scratch for the two conversions (one device status word): 256 bytes. */
BL_API size_t bitlinear_i2s_workspace_size(void);

/* Export BitLinear packed weights to I2_S.
 *   packed  device uint32 [N, K/16], D device fp32 [N] (every row the same
 *           value, as bitlinear_pack_weights writes it).
 *   i2s     device buffer of bitlinear_i2s_bytes(N, K) bytes (16-byte
 *           aligned); gets the blocks, then the scale RN(1/D[0]), which for a
 *           pack's D = mean_c is exactly the quantiser's s = RN(1/mean_c).
 * 1 <= N, K as for the forward. Synchronous: returns BL_ERR_FORMAT if a
 * packed field holds 3, the rows of D differ, or D[0] or 1/D[0] is not finite
 * and positive (the contents of i2s are then unspecified). */
BL_API int bitlinear_i2s_export(const uint32_t* packed, const float* D, int64_t N, int64_t K, int layout,
                                uint8_t* i2s, void* ws, size_t ws_bytes, bl_stream_t stream);

/* Import an I2_S buffer (device, bitlinear_i2s_bytes(N, K) bytes, 16-byte
 * aligned) into BitLinear packed weights [N, K/16] and D [N] = RN(1/scale)
 * for every row. Padding values of the tail block are ignored. Synchronous:
 * returns BL_ERR_FORMAT if a value's field holds 3 or the scale (or its
 * reciprocal) is not finite and positive (packed and D are then
 * unspecified). */
BL_API int bitlinear_i2s_import(const uint8_t* i2s, int64_t N, int64_t K, int layout,
                                uint32_t* packed, float* D, void* ws, size_t ws_bytes, bl_stream_t stream);

/* Asynchronous forms of the two conversions, for converting many tensors
 * with one check at the end: same arguments and checks, but nothing is
 * synchronised and a format error is OR-ed into the status word at the start
 * of `ws` instead of being returned. The caller zeroes that word before the
 * first call (a zero-filled workspace); bitlinear_i2s_status reads it. */
BL_API int bitlinear_i2s_export_async(const uint32_t* packed, const float* D, int64_t N, int64_t K, int layout,
                                      uint8_t* i2s, void* ws, size_t ws_bytes, bl_stream_t stream);
BL_API int bitlinear_i2s_import_async(const uint8_t* i2s, int64_t N, int64_t K, int layout,
                                      uint32_t* packed, float* D, void* ws, size_t ws_bytes, bl_stream_t stream);

/* Synchronises `stream`, reads and clears the status word of `ws`: BL_OK if
 * no asynchronous conversion since the last read met a format error, else
 * BL_ERR_FORMAT. */
BL_API int bitlinear_i2s_status(void* ws, size_t ws_bytes, bl_stream_t stream);

/* Diagnostic for the failure-detection path. Launches one thread that waits
 * on a shared-memory barrier that nothing ever completes, using the same
 * time-bounded wait as the tensor-core kernel, with a limit of limit_ns
 * (capped at 100 ms). The wait gives up, records its code in the workspace
 * error word and the kernel returns normally, so
 * bitlinear_workspace_error() then reports BL_ERR_DEVICE. No fault, trap or
 * hang is involved. Asynchronous. */
BL_API int bitlinear_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns,
                                           bl_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */
