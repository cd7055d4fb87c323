/*
 * opt2s.h -- C ABI of the B200 (sm_100a) 32-bit two-state optimizer step.
 *
 * What is computed
 * ----------------
 * One in-place update of param, state1 and state2 from a gradient, element by
 * element, with no cross-element reduction, over a collection of tensors in a
 * single kernel launch.  The method is the "32-bit two-state" optimizer update
 * of bitsandbytes issue "Investigate a 256-thread SM103 path for small 32-bit
 * optimizer tensors" (section "Problem": the kOptimizer32bit2State update with
 * fp32 state; section "Scope": decoupled weight decay applied before the
 * update; section "Correctness oracle": ADAM/AdamW and ADEMAMIX, FP16/BF16/FP32
 * param and grad storage, weight decay and skip_zeros, gradient unchanged,
 * and launch geometry must not change the arithmetic).  The formulas are the
 * standard ones: Adam (Kingma & Ba 2015, Algorithm 1), decoupled weight decay
 * (Loshchilov & Hutter 2019, Algorithm 2) and AdEMAMix (Pagliardini et al.
 * 2024, Algorithm 1).  Per element, at step t >= 1, every operation rounded
 * to fp32 in this order (no fused multiply-add, no flush-to-zero):
 *
 *     if (skip_zeros && g == 0)  leave the element wholly unchanged
 *     m   = beta1*m + (1-beta1)*g
 *     v   = beta2*v + ((1-beta2)*g)*g
 *     num = m / bc1                                   bc1 = 1 - beta1^t
 *     AdEMAMix:  m2  = beta3*m2 + (1-beta3)*g
 *                num = num + alpha*m2
 *     den = sqrt(v / bc2) + eps                       bc2 = 1 - beta2^t
 *     p   = p*decay - lr*(num/den)                    decay = 1 - lr*wd
 *
 * bc1, bc2 and decay are evaluated in double on the host and rounded to fp32
 * once.  fp16/bf16 param and grad are widened exactly; the new param is
 * narrowed with round-to-nearest-even.  State is always fp32.
 *
 * Memory layout and ownership
 * ---------------------------
 * All tensor buffers are DEVICE memory owned by the caller (e.g. allocated by
 * PyTorch), contiguous, and must stay valid until the step's work on `stream`
 * has finished.  Per tensor of `numel` elements:
 *     param   numel elements of `dtype`           read and written
 *     grad    numel elements of `dtype`           read only, never written
 *     state1  Adam: m, numel floats               read and written
 *             AdEMAMix: [m1 | m2], 2*numel floats (m2 starts at state1+numel)
 *     state2  v, numel floats                     read and written
 * State must be zero-filled by the caller before step 1.  Pointers need only
 * element alignment (torch storage offsets are fine); 16-byte alignment of all
 * arrays at the same element gives the 128-bit vector path, anything else
 * takes a scalar path with bitwise identical results.
 * The library owns only its launch tables (device memory plus host copies),
 * held by a plan; opt2s_step keeps plans in a per-device cache that
 * opt2s_release_cache() frees.
 *
 * Errors
 * ------
 * Every entry point returns OPT2S_OK (0) or a negative opt2s_status.  All
 * arguments are validated before any launch, so an argument error never
 * leaves a partial update.  OPT2S_ERR_CUDA means a CUDA call failed; the
 * CUDA error is kept in opt2s_last_cuda_error().  Calls are asynchronous with
 * respect to the host: execution errors of the kernel surface at the next
 * synchronizing CUDA call.
 */
#ifndef OPT2S_H
#define OPT2S_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* 2: opt2s_step_scalars carries the fp32 splits of the bias-correction
 * reciprocals (80 bytes a step, was 64). */
#define OPT2S_ABI_VERSION 2

/* Storage type of param and grad.  State is always fp32. */
typedef enum { OPT2S_F32 = 0, OPT2S_F16 = 1, OPT2S_BF16 = 2 } opt2s_dtype;

/* OPT2S_ADAM is Adam, and AdamW when weight_decay != 0. */
typedef enum { OPT2S_ADAM = 0, OPT2S_ADEMAMIX = 1 } opt2s_algo;

typedef enum {
    OPT2S_OK = 0,
    OPT2S_ERR_INVALID_ARG = -1, /* null pointer, bad size/dtype/algo/step, non-finite or
                                   out-of-range hyper-parameter, misaligned element */
    OPT2S_ERR_ALIAS = -2,       /* a written buffer overlaps another buffer */
    OPT2S_ERR_NO_MEMORY = -3,   /* the library could not allocate its tables */
    OPT2S_ERR_CUDA = -4,        /* a CUDA call failed (see opt2s_last_cuda_error) */
    OPT2S_ERR_DEVICE = -5,      /* plan used on another device than it was made on */
    OPT2S_ERR_TOO_LARGE = -6    /* more chunks than the launch tables can index */
} opt2s_status;

/* One tensor of the collection (all pointers are device pointers). */
typedef struct {
    void *param;
    const void *grad;
    float *state1;
    float *state2;
    int64_t numel;      /* >= 0; 0 means "skip this record" */
    int32_t dtype;      /* opt2s_dtype, for param and grad */
    int32_t reserved;   /* must be 0 */
} opt2s_tensor;

/* The collection: a HOST array of `count` records (count >= 0). */
typedef struct {
    const opt2s_tensor *tensors;
    int32_t count;
} TensorListDesc;

/* Hyper-parameters of one step.  beta1, beta2 (and beta3 for AdEMAMix) in
 * [0, 1); eps >= 0; lr, alpha, weight_decay finite; skip_zeros 0 or 1.
 * beta3 and alpha are ignored by Adam. */
typedef struct {
    float lr, beta1, beta2, beta3, alpha, eps, weight_decay;
    int32_t algo;       /* opt2s_algo */
    int32_t skip_zeros; /* 1: elements whose grad is +0 or -0 are left unchanged */
} Hyper;

/*
 * One optimizer step over the whole collection, in ONE kernel launch on
 * `stream` (0 = legacy default stream), on the current CUDA device.
 * `step` is the 1-based index t of this update (t >= 1).
 * The launch tables for `desc` come from a per-device cache keyed by the
 * descriptor's contents and the algorithm; the first call with a new
 * collection builds them (host work plus a synchronous upload), later calls
 * only launch.  An empty collection (count == 0 or all numel == 0) is a no-op.
 */
int opt2s_step(const TensorListDesc *desc, const Hyper *hyper, int step,
               cudaStream_t stream);

/*
 * Explicit plans, for callers that step the same collection many times and
 * want no per-call descriptor lookup.  opt2s_plan_create validates `desc` for
 * `algo`, builds the chunk table and uploads it to the current device
 * (synchronously).  opt2s_plan_step launches the step (hyper->algo must equal
 * the plan's algo; the current device must be the plan's device).
 * opt2s_plan_destroy waits for the device and frees the plan; NULL is a no-op.
 */
typedef struct opt2s_plan opt2s_plan;
int opt2s_plan_create(const TensorListDesc *desc, int32_t algo,
                      opt2s_plan **out_plan);
int opt2s_plan_step(const opt2s_plan *plan, const Hyper *hyper, int step,
                    cudaStream_t stream);
int opt2s_plan_destroy(opt2s_plan *plan);

/* Number of chunk records in a plan (the work units of one launch). */
int64_t opt2s_plan_num_chunks(const opt2s_plan *plan);

/*
 * Steps that a captured CUDA graph can replay.
 *
 * A captured launch keeps the arguments it was captured with, so a graph of
 * opt2s_plan_step would repeat one step number.  Here the per-step scalars
 * come from a DEVICE table instead: opt2s_fill_step_scalars computes, on the
 * host and exactly as opt2s_step does, the scalars of steps first_step ..
 * first_step+count-1; the caller uploads them to device memory.
 * opt2s_plan_step_table then launches the step with the scalars
 * d_table[*d_index] (d_index: one int32 in device memory) and a one-thread
 * kernel that advances *d_index, to -1 after the last entry; an index outside
 * [0, table_len) performs no update.  Both launches may be captured; each
 * replay performs the next step.  Results are bitwise equal to opt2s_step.
 * skip_zeros selects the kernel (0 or 1); the plan fixes the algorithm.
 * The first call for a plan should come before capture starts (it may query
 * device attributes).  Graph capture of this entry point is what the
 * bitsandbytes issue "Investigate a 256-thread SM103 path for small 32-bit
 * optimizer tensors" asks of its launch path (section "Scope": safe for CUDA
 * graph capture; section "B300 benchmark and acceptance": a graph-compatible
 * direct-call collection).
 */
typedef struct {
    float lr, beta1, beta2, beta3;
    float one_minus_beta1, one_minus_beta2, one_minus_beta3;
    float alpha, eps, bc1, bc2, decay;
    double inv_bc1, inv_bc2;    /* correctly rounded binary64 1/bc1, 1/bc2 */
    float rcp_bc1_hi, rcp_bc1_lo;   /* fp32 split of inv_bc1: RN32(inv), RN32(inv - hi) */
    float rcp_bc2_hi, rcp_bc2_lo;   /* and of inv_bc2 */
} opt2s_step_scalars;

int opt2s_fill_step_scalars(const Hyper *hyper, int first_step, int count,
                            opt2s_step_scalars *out);
int opt2s_plan_step_table(const opt2s_plan *plan, int32_t skip_zeros,
                          const opt2s_step_scalars *d_table, int32_t table_len,
                          int32_t *d_index, cudaStream_t stream);

/*
 * ZeRO-style sharded step: gradient reduce-scatter, update and parameter
 * all-gather fused in one kernel over peer memory.
 *
 * `world` ranks (<= OPT2S_MAX_WORLD) each hold the whole flat param buffer and
 * their own whole flat grad buffer (same length and storage dtype on every
 * rank), and optimizer state only for their shard.  opt2s_shard_range gives
 * rank r's shard: a contiguous range of the flat buffers, ranges disjoint and
 * covering [0, numel), balanced to within 8 elements, starts multiples of 8.
 * opt2s_shard_step, called by rank r (on its device, `stream`), updates every
 * element e of its shard with
 *     g = (g_0[e] + g_1[e] + ... + g_{world-1}[e]) / world
 * (storage values widened exactly; fp32 additions in rank order, then an fp32
 * division, each rounded once), then the plain step's update, and stores the
 * new param into EVERY rank's param buffer.  params[q] and grads[q] are rank
 * q's buffers as addressable from this rank's device (peer mappings: CUDA IPC,
 * symmetric memory, or peer access between devices of one process); state1 /
 * state2 hold this rank's shard (state1: m, or [m1 | m2] with 2 x shard
 * length floats; state2: v), zero before step 1.  Ranks never wait for one
 * another inside the kernel; the caller must order each step after every
 * rank's gradient is complete and before any rank reads params again (e.g. a
 * cross-rank barrier on both sides).  With world == 1 the result is bitwise
 * that of opt2s_step.  No TMA and no multicast touch peer memory.
 */
#define OPT2S_MAX_WORLD 8
typedef struct {
    int32_t world;
    int32_t rank;
    int64_t numel;                           /* length of every flat buffer */
    int32_t dtype;                           /* opt2s_dtype of params and grads */
    int32_t reserved;                        /* must be 0 */
    void *params[OPT2S_MAX_WORLD];           /* [q] rank q's param buffer */
    const void *grads[OPT2S_MAX_WORLD];      /* [q] rank q's grad buffer */
    float *state1;
    float *state2;
} opt2s_shard_desc;

int opt2s_shard_range(int64_t numel, int32_t world, int32_t rank, int64_t *start,
                      int64_t *len);

/*
 * Peer mappings for the sharded step between processes (one per GPU): CUDA
 * IPC.  opt2s_ipc_export gives the handle of the device allocation that
 * holds `ptr` and ptr's byte offset inside it; another process passes both to
 * opt2s_ipc_open, which maps the allocation (enabling peer access on first
 * use when it lives on another GPU of the node) and returns its base and the
 * mapped address of the exporter's `ptr`.  opt2s_ipc_close(base) unmaps it
 * (only after every kernel that uses the mapping has finished).  A handle
 * is 64 opaque bytes; it is valid while the exporting allocation lives.
 * Errors: OPT2S_ERR_INVALID_ARG for null arguments, OPT2S_ERR_CUDA (with
 * opt2s_last_cuda_error) when the driver refuses, e.g. for an address that is
 * not device memory or a handle opened in the process that exported it.
 */
typedef struct {
    unsigned char bytes[64];
} opt2s_ipc_handle;

int opt2s_ipc_export(const void *ptr, opt2s_ipc_handle *handle, int64_t *offset);
int opt2s_ipc_open(const opt2s_ipc_handle *handle, int64_t offset, void **base, void **ptr);
int opt2s_ipc_close(void *base);
int opt2s_shard_step(const opt2s_shard_desc *desc, const Hyper *hyper, int step,
                     cudaStream_t stream);

/*
 * opt2s_step without any allocation by the library.  The paper this library
 * follows has no counterpart to it: it exists for callers that cannot let a
 * library allocate device memory -- runtimes that own all device memory
 * through their own pool, deployments whose memory footprint is fixed at
 * start-up, or code that must avoid the implicit synchronization of
 * cudaMalloc/cudaFree.  Same arguments, arithmetic and results as opt2s_step.
 *
 * It calls no cudaMalloc, cudaFree or allocating library routine and keeps
 * no plan.  Each call builds the chunk table in a fixed host array and
 * uploads it with cudaMemcpyAsync on `stream` (the copy and the launch are
 * ordered on `stream` like any other work there) into a fixed device array of
 * opt2s_noalloc_max_chunks() records (65,536 records = 3 MiB), which every
 * GPU that loads the library holds until the process exits.  A collection
 * needing more chunk records (8,192 elements per chunk; at least one per
 * non-empty tensor) returns OPT2S_ERR_TOO_LARGE before any work.
 * All calls on a device share that array and leave the last call's table in
 * it; every call rewrites what it reads, so nothing must start at zero.  Calls
 * whose work overlaps on the GPU (unordered streams) race on the array.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it.
 * Calls from several host threads are serialized.  Each successful call
 * counts one kernel launch.  CUDA failures are kept in opt2s_last_cuda_error.
 */
int opt2s_step_noalloc(const TensorListDesc *desc, const Hyper *hyper, int step,
                       cudaStream_t stream);

/* Capacity of opt2s_step_noalloc's fixed chunk table, in records. */
int64_t opt2s_noalloc_max_chunks(void);

/*
 * The step with each tensor's update norm bounded: bitsandbytes' max_unorm
 * option of the same two-state update (the issue's section "Scope" keeps its
 * kernel for "max-unorm/LAMB use", and section "Correctness oracle" runs
 * "max_unorm > 0" controls).  The pages name the option without its
 * arithmetic; this library reads it as a bound on the norm of a tensor's
 * update relative to the norm of its weights:
 *
 *     u_i = num_i/den_i, the update direction of element i in the step above
 *           (0 for an element skip_zeros leaves alone)
 *     U   = sqrt(sum_i u_i^2),  P = sqrt(sum_i p_i^2), p before the step,
 *           over each tensor of the collection; binary64 squares and sums
 *     s   = max_unorm*P/U if U > max_unorm*P, else 1  (binary64, rounded to
 *           fp32 once)
 *     p_i = p_i*decay - lr*(s*u_i), with m, v (and m2) as in the step above.
 *
 * s = 1 gives exactly opt2s_step's bits.  The sums have a fixed order (lane
 * l of a warp adds elements l, l+32, ... of a 2,048-element block, then a
 * fixed tree over lanes; a group's blocks and a tensor's groups are added
 * in fixed orders too),
 * so s does not depend on launch geometry or storage alignment; against a
 * plain sequential binary64 sum it can differ only when the ratio lies
 * within a few binary64 ulp of an fp32 rounding boundary.
 *
 * max_unorm: finite and > 0 (else OPT2S_ERR_INVALID_ARG).  Other arguments
 * and validation as opt2s_step.  Four launches on `stream`: the sums per
 * 2,048-element block, the sums per group of 64 blocks, the per-tensor
 * scales, and the scaled update.  The tensor is read twice (once for the
 * sums, once for the update).  Plans are cached like opt2s_step's, each with
 * a workspace of 64 bytes per 2,048 elements plus 24 bytes per group and
 * 8 bytes per tensor and per chunk, freed by opt2s_release_cache().  The
 * workspace belongs to the collection's plan: like its params and states,
 * two steps of the same collection must not overlap on the GPU.
 */
int opt2s_step_max_unorm(const TensorListDesc *desc, const Hyper *hyper, float max_unorm,
                         int step, cudaStream_t stream);

/*
 * LAMB: the layer-wise adaptive step of You et al., "Large Batch Optimization
 * for Deep Learning: Training BERT in 76 minutes", ICLR 2020, Algorithm 2,
 * with each tensor of the collection as a layer.  The issue's section "Scope"
 * keeps the two-state kernel for "max-unorm/LAMB use" without writing LAMB
 * out; this library follows Algorithm 2 with the scaling function phi the
 * identity:
 *
 *     u_i = num_i/den_i, the Adam direction of element i in the step above
 *     w_i = u_i + weight_decay*p_i                  (fp32; 0 for an element
 *                                                    skip_zeros leaves alone)
 *     W   = sqrt(sum_i w_i^2),  P = sqrt(sum_i p_i^2), p before the step,
 *           per tensor, in binary64
 *     r   = P/W if P > 0 and W > 0, else 1 (binary64, rounded to fp32 once)
 *     p_i = p_i - lr*(r*w_i), with m and v as in the step above.
 *
 * The weight decay is inside the trust-ratio scaled update (Algorithm 2),
 * not applied first as in opt2s_step; bc1, bc2 as in opt2s_step.
 * hyper->algo must be OPT2S_ADAM (else OPT2S_ERR_INVALID_ARG).  Sums have
 * the fixed order of opt2s_step_max_unorm, so r does not depend on launch
 * geometry or alignment.  Four launches on `stream`; the plans, tables and
 * workspace are those of opt2s_step_max_unorm (shared cache entries), with
 * the same rule that two steps of the same collection must not overlap on
 * the GPU.  Other arguments and validation as opt2s_step.
 */
int opt2s_step_lamb(const TensorListDesc *desc, const Hyper *hyper, int step,
                    cudaStream_t stream);

/*
 * 8-bit blockwise optimizer state, for collections whose tensors of at least
 * min_8bit_size elements keep their state in 8 bits and whose smaller tensors
 * keep it in fp32 -- the routing the issue's section "Problem" describes for
 * bitsandbytes' 8-bit Adam/AdamW/AdEMAMix (min_8bit_size = 4096 by default):
 * the small bias/norm/adapter tensors take the 32-bit update.  Both kinds are
 * stepped in ONE launch.
 *
 * The 8-bit format is that of Dettmers, Lewis, Shleifer & Zettlemoyer,
 * "8-bit Optimizers via Block-wise Quantization", ICLR 2022: each state
 * quantity of a tensor is cut into blocks of OPT2S_BLOCK8 = 2048 elements
 * (section 2.1); a block keeps one fp32 absmax and one byte per element, the
 * code of a value of a 256-entry map -- dynamic tree quantization for the
 * signed m and m2 (section 2.2), dynamic quantization for the non-negative v
 * (section 2.3).  Code c stands for the c-th smallest map value.  The maps:
 * for E = 0..6 and F = 6 - E (signed) or 7 - E (unsigned), the values
 * 10^-E * (0.1 + 0.9*(2f+1)/2^(F+1)), f = 0 .. 2^F - 1 (both signs in the
 * signed map), each rounded to fp32 once, plus 0 and 1.0: 256 values each.
 *
 * Per 8-bit block and step: every element's m = map_s[code]*absmax (fp32
 * product), likewise v (map_u) and m2; the update of opt2s_step on these
 * values; then each quantity's new block absmax max|x| and new codes: the
 * code of the map value nearest to x/absmax (fp32 division; an exact tie
 * takes the lower code), or the code of 0 when the absmax is 0.  With
 * skip_zeros an element whose gradient is zero keeps its param and its
 * dequantized state, which is requantized with the block's new absmax.
 * A 32-bit record is stepped exactly as opt2s_step steps it.
 *
 * Per record, by state_bits:
 *   8:  state1  uint8 codes of m (numel bytes), AdEMAMix [m1 | m2] (2*numel)
 *       state2  uint8 codes of v (numel bytes)
 *       absmax1 fp32 absmax of m per block (nb = ceil(numel/2048) floats),
 *               AdEMAMix [m1 absmaxes | m2 absmaxes] (2*nb)
 *       absmax2 fp32 absmax of v per block (nb floats)
 *       Zero state before step 1: every absmax 0 (the codes then do not
 *       matter; zero-filling everything is fine).
 *   32: state1, state2 fp32 as in opt2s_tensor; absmax1, absmax2 NULL.
 * Pointers need element alignment (fp32 state and absmaxes: 4 bytes; codes:
 * none); aligned full blocks take 16-byte and 8-byte accesses.
 *
 * opt2s_step_8bit: one step of the collection in one launch on `stream`, one
 * CTA per 8-bit block, warps on the 32-bit tensors' chunks.  Plans (the
 * block and chunk tables) are cached per device like opt2s_step's.
 * Validation as opt2s_step, plus state_bits in {8, 32}, non-null absmax
 * pointers exactly for 8-bit records, and no overlap of any written buffer
 * (codes and absmaxes included) with another buffer.
 */
#define OPT2S_BLOCK8 2048
#define OPT2S_MIN_8BIT_SIZE 4096

typedef struct {
    void *param;
    const void *grad;
    void *state1;
    void *state2;
    float *absmax1;
    float *absmax2;
    int64_t numel;
    int32_t dtype;        /* opt2s_dtype of param and grad */
    int32_t state_bits;   /* 8 or 32 */
} opt2s_tensor8;

typedef struct {
    const opt2s_tensor8 *tensors;   /* HOST array of `count` records */
    int32_t count;
} TensorListDesc8;

int opt2s_step_8bit(const TensorListDesc8 *desc, const Hyper *hyper, int step,
                    cudaStream_t stream);

/* The routing: 8 when numel >= min_8bit_size, else 32 (min_8bit_size <= 0
 * means OPT2S_MIN_8BIT_SIZE). */
int opt2s_8bit_state_bits(int64_t numel, int64_t min_8bit_size);

/* Frees every cached plan of every device (waits for the devices first). */
int opt2s_release_cache(void);

/* Human-readable text for a status code (static storage). */
const char *opt2s_error_string(int status);

/* The cudaError_t of the last failed CUDA call in this thread (0 if none). */
int opt2s_last_cuda_error(void);

/* OPT2S_ABI_VERSION of the loaded library. */
int opt2s_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OPT2S_H */
