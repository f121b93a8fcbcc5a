/*
 * mole.h -- C ABI of libmole, the B200 (sm_100a) implementation of the
 * Mixture-of-Lookup-Experts (MoLE) inference lookup path.
 *
 * Source page ("MoLE page"): "ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE，
 * 内存搬运代价降低1000倍" (zejuncao.github.io, 2025-05-07).  The page states the
 * method in prose only (its formulas and figures were lost); the readings this
 * library takes are stated at each entry point.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, row-major and
 *     contiguous.  The library never frees or retains them.
 *   - Work is enqueued asynchronously on `stream` (0 = legacy default stream).
 *     Argument errors are detected on the host and returned synchronously;
 *     nothing is launched then.
 *   - Errors detected on the device (a token id outside [0, V), a wait that ran
 *     out of time) set a per-device error word; `mole_check` reads and clears
 *     it.  A token with a bad id gets a NaN output row.
 *   - The library allocates no device memory of its own apart from static
 *     per-device variables (the error word, and the fixed scratch array of
 *     mole_build_lut_noalloc).  Scratch memory, where the other entry points
 *     need it, is passed in by the caller.
 *   - bf16 tensors are IEEE bfloat16 bit patterns; fp16 scales are IEEE binary16.
 */
#ifndef MOLE_H_
#define MOLE_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOLE_OK = 0,
  MOLE_ERR_ARG = 1,          /* bad pointer, size or enum value */
  MOLE_ERR_ALIGN = 2,        /* a pointer is not 16-byte aligned where required */
  MOLE_ERR_UNSUPPORTED = 3,  /* valid but unsupported shape (see each call) */
  MOLE_ERR_WORKSPACE = 4,    /* scratch buffer missing or too small */
  MOLE_ERR_INDEX = 5,        /* (mole_check) a token id was outside [0, V) */
  MOLE_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed */
  MOLE_ERR_TIMEOUT = 7,      /* (mole_check) host wait or device wait ran out */
  MOLE_ERR_NO_DEVICE = 8     /* no sm_100 device current */
} mole_status;

typedef enum { MOLE_F32 = 0, MOLE_BF16 = 1 } mole_dtype;

typedef enum {
  MOLE_ACT_GELU_ERF = 0,   /* x * Phi(x) (default reading of "GELU FFN") */
  MOLE_ACT_GELU_TANH = 1,  /* tanh approximation of GELU */
  MOLE_ACT_RELU = 2,
  MOLE_ACT_SILU = 3,
  MOLE_ACT_IDENTITY = 4
} mole_act;

/* Human-readable name of a status code (static storage). */
const char* mole_status_str(mole_status s);

/* Library version, major * 10000 + minor * 100 + patch. */
int mole_version(void);

/*
 * ---- Reparameterisation: build the lookup table (MoLE page, 推理阶段) ----
 *
 * Feeds the embedding matrix to every routed expert:
 *     LUT[v, j, :] = f_j(E[v, :]),   f_j(x) = act(x . W1[j]) . W2[j]
 * (expert form and activation are this library's reading; the page prints no
 * formula).  All routed experts are evaluated; the experts can be dropped
 * afterwards.
 *
 *   embed : [V, D]       dt
 *   W1    : [N, D, Dr]   dt
 *   W2    : [N, Dr, D]   dt
 *   lut   : [V, N, D]    dt  (output; token v's N rows are contiguous)
 *   workspace: scratch for the expert hidden activations H = act(E . W1[j]);
 *     at least mole_build_lut_workspace(...) bytes for one expert at a time,
 *     more lets several experts run per launch (up to all N).  Contents on
 *     return are unspecified.
 * dt == MOLE_BF16: bf16 in, fp32 accumulate on the tcgen05 tensor cores, H
 *   rounded to bf16, bf16 out.  Tensor-core path needs D % 64 == 0 and
 *   Dr % 64 == 0 and 16-byte aligned pointers; other shapes use a CUDA-core path.
 * dt == MOLE_F32: fp32 throughout on CUDA cores.
 * Returns MOLE_ERR_WORKSPACE if ws_bytes is below the one-expert minimum.
 */
size_t mole_build_lut_workspace(int64_t V, int64_t D, int32_t N, int64_t Dr, mole_dtype dt,
                                int32_t experts_per_launch);
mole_status mole_build_lut(const void* embed, const void* W1, const void* W2, int64_t V,
                           int64_t D, int32_t N, int64_t Dr, mole_act act, mole_dtype dt,
                           void* lut, void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * mole_build_lut without caller-provided scratch, for callers that cannot
 * allocate device memory when they build a table: serving loops that allow no
 * device allocation after start-up (their memory footprint is fixed up
 * front), and plugin hosts that own all device memory and give plugins no
 * allocator.  The MoLE page has no counterpart; it is an interface
 * convenience.
 *
 * Same arguments, layouts and results as mole_build_lut, minus the workspace:
 * the hidden activations of each group of experts live in a fixed 16 MiB array
 * in this library's device memory (held by every GPU that loads the library
 * until the process exits).  One expert's activations, V * Dr * (2 bytes for
 * bf16, 4 for fp32), must fit in it, else MOLE_ERR_WORKSPACE and nothing is
 * launched; experts are built in groups of as many as fit.  The first call on
 * each device looks the array's device address up (cudaGetSymbolAddress, with
 * that device current), and looks it up again after the device's context has
 * changed (a device reset); make that first call before any stream capture.
 * Every call uses the same array, which keeps the last call's contents: calls
 * that overlap on the GPU (other streams, other threads) race on it.  The
 * array needs no clearing between calls (each expert's activations are
 * written before they are read).  No device memory is allocated or freed.
 */
mole_status mole_build_lut_noalloc(const void* embed, const void* W1, const void* W2, int64_t V,
                                   int64_t D, int32_t N, int64_t Dr, mole_act act, mole_dtype dt,
                                   void* lut, cudaStream_t stream);

/*
 * ---- Lookup-combine (MoLE page, 训练阶段 + 推理阶段) ----
 *
 * For each token t (router on the hidden state, all N routed experts active,
 * rows fetched by direct addressing on the token id):
 *     z_j = sum_d h[t, d] Wr[d, j]          (fp32 accumulate)
 *     g   = softmax(z)                        (max-subtracted, fp32)
 *     out[t, :] = sum_j g_j LUT[ids[t], j, :]  (fp32 accumulate)
 * Only the routed-expert mixture is produced; shared experts and the residual
 * are the caller's.
 *
 *   ids : [T] int32 in [0, V)    h : [T, D] dt    Wr : [D, N] dt
 *   lut : [V, N, D] dt           out : [T, D] fp32 (overwritten)
 * dt == MOLE_BF16 needs D % 16 == 0, N <= 32 and 16-byte aligned h, lut, out.
 * dt == MOLE_F32 needs D % 4 == 0, N <= 32 and 16-byte aligned h, lut, out.
 * T == 0 is a no-op.  A token with ids[t] outside [0, V) gets a NaN row and
 * sets the device error word (MOLE_ERR_INDEX from mole_check).
 */
mole_status mole_lookup_combine(const int32_t* ids, int64_t T, const void* h, const void* Wr,
                                const void* lut, int64_t V, int32_t N, int64_t D,
                                mole_dtype dt, float* out, cudaStream_t stream);

/*
 * ---- Token groups: the combine with each distinct row block read once ----
 * (MoLE page, 复杂度分析: a token's traffic is its N expert-output rows; a batch
 * that repeats an id needs that id's rows only once.  推理阶段: every MoLE
 * layer indexes its table with the same input token ids, so one grouping of
 * the batch serves all layers.)
 *
 * mole_token_groups_build groups the batch's tokens by id into `groups`, a
 * caller-owned device buffer of at least mole_token_groups_workspace(T, N)
 * bytes, 16-byte aligned (N = the experts of the layers it will serve).  Its
 * contents are opaque; the grouping stays valid until the buffer is rebuilt.
 * Ids outside [0, V) are left out of every group and set the device error
 * word (MOLE_ERR_INDEX).  One cooperative kernel launch (all of its CTAs
 * resident at once), then one plain launch that lists each SM's share of the
 * work for the per-layer kernels; the grouping therefore belongs to the
 * device it was built on (a layer call on a device with another SM count
 * writes no output and mole_check reports MOLE_ERR_ARG).
 *
 * mole_lookup_combine_groups is mole_lookup_combine (same arguments, layouts,
 * results bit for bit, and error behaviour) for a batch whose grouping was
 * built from the same ids, T and N: each distinct id's row block is read once
 * and applied to all of that id's tokens.  The call may also write one
 * layer's gates into `groups`, so calls that share a groups buffer must not
 * overlap on the GPU.  The grouped kernels serve bf16 inputs with T >= 1024;
 * other calls run the mole_lookup_combine kernels (the grouping is then
 * unused).
 *
 * mole_lookup_combine_grouped builds the grouping in `workspace` and runs
 * mole_lookup_combine_groups, for a single layer;
 * mole_lookup_combine_grouped_workspace equals mole_token_groups_workspace.
 * All three return MOLE_ERR_WORKSPACE if the buffer is NULL or too small
 * (T > 0) and MOLE_ERR_ALIGN if it is not 16-byte aligned.
 */
size_t mole_token_groups_workspace(int64_t T, int32_t N);
mole_status mole_token_groups_build(const int32_t* ids, int64_t T, int64_t V, int32_t N, void* groups,
                                    size_t bytes, cudaStream_t stream);
mole_status mole_lookup_combine_groups(const int32_t* ids, int64_t T, const void* groups, size_t bytes,
                                       const void* h, const void* Wr, const void* lut, int64_t V, int32_t N,
                                       int64_t D, mole_dtype dt, float* out, cudaStream_t stream);
size_t mole_lookup_combine_grouped_workspace(int64_t T, int32_t N);
mole_status mole_lookup_combine_grouped(const int32_t* ids, int64_t T, const void* h, const void* Wr,
                                        const void* lut, int64_t V, int32_t N, int64_t D, mole_dtype dt,
                                        float* out, void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * ---- NF3 table compression (MoLE page, 实验结果: 3-bit table, e.g. NF3) ----
 *
 * Quantises a bf16 table [V, N, D] (D % 64 == 0) in blocks of 64 consecutive
 * elements of one (v, j) row, in IEEE fp32:
 *     s = fp16(min(max_e |x_e|, 65504))                 (ties to even)
 *     c_e = #{k : x_e / s > mid_k}   (s > 0; correctly rounded division)
 *     c_e = 3 (the level 0.0)        (s == 0)
 * with the NormalFloat k=3 levels (QLoRA construction, rounded to fp16; see
 * mole_nf3_levels) and mid_k the fp32 midpoints of adjacent levels.  Code e
 * occupies bits [3e, 3e+3) of the block's 24-byte little-endian bit string.
 *   codes  : [V, N, D/64, 24] uint8    scales : [V, N, D/64] fp16 bits
 * lut_bf16 must be 16-byte aligned; codes 8-byte aligned.
 */
mole_status mole_quantize_lut_nf3(const void* lut_bf16, int64_t V, int32_t N, int64_t D,
                                  uint8_t* codes, uint16_t* scales, cudaStream_t stream);

/*
 * mole_build_lut and mole_quantize_lut_nf3 in one pass: the bf16 table is
 * never written.  The second tensor-core GEMM's epilogue rounds each output
 * to bf16 (the value mole_build_lut would store), quantises every 64-element
 * block of a (v, j) row in registers and writes the codes and the fp16 scale;
 * the results equal mole_build_lut followed by mole_quantize_lut_nf3, bit for
 * bit.  bf16 only, on the tensor-core path (D % 64 == 0, Dr % 64 == 0,
 * 16-byte aligned embed, W1, W2 and workspace; else MOLE_ERR_UNSUPPORTED);
 * codes 8-byte aligned.  Workspace as for mole_build_lut (dt = MOLE_BF16).
 */
mole_status mole_build_lut_nf3(const void* embed, const void* W1, const void* W2, int64_t V, int64_t D,
                               int32_t N, int64_t Dr, mole_act act, uint8_t* codes, uint16_t* scales,
                               void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * mole_lookup_combine over an NF3 table: the row element for (id, j, d) is
 * level[c] * s of its block (exact in fp32), dequantised in registers inside
 * the gather.  Same arguments and error behaviour as mole_lookup_combine,
 * with D % 64 == 0.
 */
mole_status mole_lookup_combine_nf3(const int32_t* ids, int64_t T, const void* h,
                                    const void* Wr, const uint8_t* codes,
                                    const uint16_t* scales, int64_t V, int32_t N, int64_t D,
                                    mole_dtype dt, float* out, cudaStream_t stream);

/*
 * mole_lookup_combine_nf3 for a batch whose token grouping was built from the
 * same ids, T and N (see mole_token_groups_build): each distinct id's code and
 * scale blocks are read and decoded once and applied to all of that id's
 * tokens.  Same arguments, results (bit for bit) and error behaviour as
 * mole_lookup_combine_nf3, plus the groups buffer (as for
 * mole_lookup_combine_groups).  The grouped kernels serve bf16 inputs,
 * T >= 1024, N <= 16 with N * D/64 a multiple of 8, and 16-byte aligned codes
 * and scales; other calls run the mole_lookup_combine_nf3 kernels.
 */
mole_status mole_lookup_combine_nf3_groups(const int32_t* ids, int64_t T, const void* groups, size_t bytes,
                                           const void* h, const void* Wr, const uint8_t* codes,
                                           const uint16_t* scales, int64_t V, int32_t N, int64_t D, mole_dtype dt,
                                           float* out, cudaStream_t stream);

/*
 * ---- Offloaded table (MoLE page, 推理阶段 and 复杂度分析) ----
 *
 * The page's deployment: the table lives in slower, larger memory (CPU memory
 * or storage) and per token only its N expert-output rows move to the
 * accelerator.  Here the table (or its NF3 codes and scales) stays in host
 * memory that is pinned and mapped into the device's address space
 * (cudaHostAlloc, or cudaHostRegister with cudaHostRegisterMapped; memory of
 * the current device is accepted too).  Per batch each distinct id's row
 * block crosses the link once, into a device staging buffer, and the combine
 * reads the staging buffer.  Both calls take a grouping of the batch built by
 * mole_token_groups_build (same T, V and N): it numbers the batch's distinct
 * ids 0..U-1, and the staging buffer holds the row block of distinct id u at
 * index u.
 *
 * mole_offload_staging_bytes: size of the staging buffer for a batch of T
 *   tokens over a table of V ids (room for min(T, V) row blocks).  nf3 = 0:
 *   the table has dtype dt, [V, N, D]; nf3 = 1: NF3 codes [V, N, D/64, 24]
 *   and fp16 scales [V, N, D/64] (D % 64 == 0).  0 for invalid arguments.
 *
 * mole_offload_stage copies the batch's distinct row blocks from `table`
 *   (and, NF3, `scales`) into `staging` (device, 16-byte aligned, at least
 *   mole_offload_staging_bytes bytes).  table must be 16-byte aligned (NF3
 *   codes 8-byte, scales 2-byte).  If n_rows is not NULL it receives U (one
 *   device int32).  Pageable (unregistered) host memory gives MOLE_ERR_ARG.
 *   One kernel launch; the host table must stay unchanged until it has run.
 *
 * mole_lookup_combine_offload is mole_lookup_combine (or, nf3 = 1,
 *   mole_lookup_combine_nf3) over the staged rows: the same results, bit for
 *   bit, as those calls on the table itself, and the same error behaviour
 *   (a token whose id is outside [0, V) gets a NaN row).  No ids argument:
 *   the grouping holds each token's dense index.  Calls that share a groups
 *   buffer must not overlap on the GPU (the call writes the layer's gates
 *   into it); a staging buffer may be refilled for the next layer once the
 *   combine that reads it has run, so two staging buffers let the next
 *   layer's copy overlap this layer's combine.
 *
 * Both return MOLE_ERR_WORKSPACE for a missing or too small groups or staging
 * buffer; T == 0 is a no-op.
 */
size_t mole_offload_staging_bytes(int64_t T, int64_t V, int32_t N, int64_t D, mole_dtype dt, int32_t nf3);
mole_status mole_offload_stage(int64_t T, const void* groups, size_t bytes, const void* table,
                               const uint16_t* scales, int64_t V, int32_t N, int64_t D, mole_dtype dt,
                               int32_t nf3, void* staging, size_t staging_bytes, int32_t* n_rows,
                               cudaStream_t stream);
mole_status mole_lookup_combine_offload(int64_t T, const void* groups, size_t bytes, const void* h,
                                        const void* Wr, const void* staging, size_t staging_bytes, int64_t V,
                                        int32_t N, int64_t D, mole_dtype dt, int32_t nf3, float* out,
                                        cudaStream_t stream);

/*
 * ---- FFN block: shared expert + routed-expert mixture + residual ----
 * (MoLE page, 训练阶段 and 推理阶段: the shared experts stay dense FFNs on the
 * previous layer's output at inference; only the routed experts become the
 * table.  The page gives no formula; this library's reading: one shared
 * expert of the routed experts' form, act(h . W1s) . W2s, and the block's
 * output is residual + shared expert + routed mixture.)
 *
 * mole_shared_ffn: out = act(h . W1s) . W2s + add + residual  (fp32)
 *   h : [T, D] bf16   W1s : [D, Ds] bf16   W2s : [Ds, D] bf16
 *   add, residual : [T, D] fp32 or NULL   out : [T, D] fp32 (may be add or
 *   residual: each element is read before it is written)
 *   Two tcgen05 GEMMs (fp32 accumulate); the hidden activation is rounded to
 *   bf16 in `workspace` (at least mole_shared_ffn_workspace(T, Ds) bytes);
 *   the additions happen in the second GEMM's epilogue.  Needs D % 64 == 0,
 *   Ds % 64 == 0 and 16-byte aligned pointers (else MOLE_ERR_UNSUPPORTED /
 *   MOLE_ERR_ALIGN).
 *
 * mole_ffn_block: out = residual + act(h . W1s) . W2s + sum_j g_j LUT[ids[t], j]
 *   The routed mixture is mole_lookup_combine_groups over `groups` (built from
 *   the same ids, T and N), written into the workspace and added in the
 *   shared expert's second GEMM epilogue.  bf16 inputs, D % 64 == 0,
 *   Ds % 64 == 0; workspace of mole_ffn_block_workspace(T, D, Ds) bytes; out
 *   may be residual.  Bad ids: NaN rows and MOLE_ERR_INDEX from mole_check,
 *   as for the combine.
 */
size_t mole_shared_ffn_workspace(int64_t T, int64_t Ds);
mole_status mole_shared_ffn(const void* h, const void* W1s, const void* W2s, int64_t T, int64_t D, int64_t Ds,
                            mole_act act, const float* add, const float* residual, float* out, void* workspace,
                            size_t ws_bytes, cudaStream_t stream);
size_t mole_ffn_block_workspace(int64_t T, int64_t D, int64_t Ds);
mole_status mole_ffn_block(const int32_t* ids, int64_t T, const void* groups, size_t groups_bytes, const void* h,
                           const void* Wr, const void* lut, int64_t V, int32_t N, const void* W1s, const void* W2s,
                           int64_t D, int64_t Ds, mole_act act, const float* residual, float* out,
                           void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * ---- Training: one MoLE layer forward and backward (MoLE page, 训练阶段) ----
 *
 * In training the routed experts take the token's embedding row as input and
 * all N are active, mixed by the router on the previous layer's output h:
 *     out[t] = sum_j softmax(h[t] . Wr)_j f_j(E[ids[t]]),
 *     f_j(x) = act(x . W1[j]) . W2[j]   (hidden activation rounded to bf16)
 * A routed expert's output depends only on the token id, so the forward
 * evaluates the experts on the batch's distinct ids only (the table build on
 * those embedding rows, tcgen05 GEMMs) and mixes them with the combine
 * kernels: `out` equals mole_lookup_combine over a table built by
 * mole_build_lut, bit for bit.  The grouping (`groups`, from
 * mole_token_groups_build with the same ids, T, V and N) supplies the distinct
 * ids.  The forward reads their count back to the host (one stream
 * synchronisation) and returns it in *n_distinct; the backward takes it back.
 *
 * mole_train_backward adds (+=, fp32) the gradients of L = sum(out * dout)
 * (dout [T, D] fp32) to dh [T, D], dWr [D, N], dE [V, D] (the batch's rows
 * only), dW1 [N, D, Dr] and dW2 [N, Dr, D]; any of them may be NULL.  The
 * backward GEMMs (bf16 operands, fp32 accumulation) run in cuBLAS, whose
 * handle (created on a device's first backward call) holds cuBLAS's own device
 * memory; its operands dL/dY and dL/dpre are rounded to bf16 from fp32.  The
 * bf16 rounding of the hidden activation counts as identity in the backward.
 * Tokens with an id outside [0, V) get NaN outputs (MOLE_ERR_INDEX from
 * mole_check) and contribute no gradient.
 *
 *   h [T, D] bf16, Wr [D, N] bf16, E [V, D] bf16, W1 [N, D, Dr] bf16,
 *   W2 [N, Dr, D] bf16; out [T, D] fp32.  D % 64 == 0, Dr % 64 == 0, N <= 32,
 *   16-byte aligned pointers.  `cache` (device, 16-byte aligned) carries the
 *   forward's intermediates to the backward: at least
 *   mole_train_cache_bytes(T, V, N, D, Dr) bytes (room for min(T, V) distinct
 *   ids), not to be reused between a step's forward and backward.
 */
size_t mole_train_cache_bytes(int64_t T, int64_t V, int32_t N, int64_t D, int64_t Dr);
mole_status mole_train_forward(const int32_t* ids, int64_t T, const void* groups, size_t groups_bytes,
                               const void* h, const void* Wr, const void* E, const void* W1, const void* W2,
                               int64_t V, int32_t N, int64_t D, int64_t Dr, mole_act act, float* out, void* cache,
                               size_t cache_bytes, int32_t* n_distinct, cudaStream_t stream);
mole_status mole_train_backward(const int32_t* ids, int64_t T, const void* groups, size_t groups_bytes,
                                const void* h, const void* Wr, const void* E, const void* W1, const void* W2,
                                int64_t V, int32_t N, int64_t D, int64_t Dr, mole_act act, const float* dout,
                                void* cache, size_t cache_bytes, int32_t n_distinct, float* dh, float* dWr,
                                float* dE, float* dW1, float* dW2, cudaStream_t stream);

/* The 8 NF3 levels as fp16 bit patterns (ascending; index 3 is 0.0) and the 7
 * fp32 decision midpoints.  Host-only; no device work. */
void mole_nf3_levels(uint16_t levels_f16[8]);
void mole_nf3_midpoints(float mid[7]);

/*
 * ---- Gather plan (the set of table rows a batch fetches; MoLE page, 复杂度分析) ----
 *
 * uniq[0..n_uniq) receives the distinct ids of the batch in ascending order,
 * slot[t] the index of ids[t] in uniq.  uniq has capacity T; n_uniq is one
 * device int32.  Needs V <= 524288 (the id set is kept on chip).  Ids outside
 * [0, V) are skipped (slot = -1) and set the device error word.
 */
mole_status mole_gather_plan(const int32_t* ids, int64_t T, int64_t V, int32_t* uniq,
                             int32_t* n_uniq, int32_t* slot, cudaStream_t stream);

/*
 * ---- Cross-layer row prefetch (MoLE page, 推理阶段 + 复杂度分析) ----
 *
 * Every MoLE layer indexes its own table with the step's input token ids, so
 * all layers' rows are known before the first layer runs.  For each of the
 * n_tables tables and each token t with 0 <= ids[t] < V, asks the GPU's L2
 * cache to fetch row ids[t] of that table (row_bytes bytes at
 * tables[l] + ids[t] * row_bytes): bulk L2 prefetches, issued from many SMs,
 * that move no data into the SMs and that nothing waits for.  Later calls
 * that read those rows (the layers' combines, in this stream or another)
 * then hit L2 while the rows stay resident (126 MB of L2: prefetch no more
 * than fits).  Results of every call are unchanged; this is a hint.
 *
 *   ids    : [T] int32 device; ids outside [0, V) are skipped (the combine
 *            that reads them reports them)
 *   tables : HOST array of n_tables (<= 64) device pointers, 16-byte aligned;
 *            an NF3 table is two tables (codes, row_bytes = N * D / 64 * 24;
 *            scales, row_bytes = N * D / 64 * 2)
 *   row_bytes : bytes of one row, a multiple of 16 (bf16 table: N * D * 2)
 * MOLE_ERR_ALIGN for unaligned tables or row_bytes, MOLE_ERR_UNSUPPORTED for
 * more than 64 tables.  T == 0 or n_tables == 0 is a no-op.
 */
mole_status mole_prefetch_rows(const int32_t* ids, int64_t T, const void* const* tables, int32_t n_tables,
                               int64_t V, int64_t row_bytes, cudaStream_t stream);

/*
 * Waits (polling, at most timeout_ms >= 0 milliseconds) for `stream` to drain,
 * then reads and clears this device's error word.  A negative timeout_ms is
 * rejected with MOLE_ERR_ARG (no host wait is unbounded).  Returns MOLE_OK,
 * MOLE_ERR_INDEX (bad token id), MOLE_ERR_TIMEOUT (stream still busy, or a
 * device-side wait gave up), MOLE_ERR_ARG (a grouping was used on a device
 * with another SM count than the one it was built on; the layer's output was
 * not written), or MOLE_ERR_CUDA (an asynchronous CUDA error).
 */
mole_status mole_check(cudaStream_t stream, int timeout_ms);

#ifdef __cplusplus
}
#endif

#endif /* MOLE_H_ */
