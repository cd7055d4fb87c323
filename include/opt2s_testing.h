/*
 * opt2s_testing.h -- validation scaffolding for the test suite.  NOT part of
 * the public API.
 *
 * bitsandbytes issue "Investigate a 256-thread SM103 path for small 32-bit
 * optimizer tensors", section "Scope", allows experimental forcing only in
 * validation scaffolding, never as a public API; these entry points are that
 * scaffolding.  They let the tests (a) run the host-side validation and
 * chunk-table builder without a GPU and (b) force other launch geometries, to
 * check the issue's "Correctness oracle" requirement that the launch geometry
 * must not change the optimizer arithmetic (results must be bitwise equal).
 *
 * The host-only queries below are exported by the library.  The forcing
 * knobs (opt2s_testing_set_chunk_elems, opt2s_testing_set_launch), the fault
 * injection (opt2s_testing_fail_allocs) and the division check
 * (opt2s_testing_check_division) exist only in the test build of the
 * library, libopt2s_testing.so (the same kernels, compiled once and linked
 * into both); the product libopt2s.so does not export them, and its launch
 * geometry cannot be changed.
 *
 * All knobs are process-wide, apply to plans created or launched afterwards,
 * and are not thread-safe against concurrent steps.
 */
#ifndef OPT2S_TESTING_H
#define OPT2S_TESTING_H

#include "opt2s.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One work unit of a launch as the host builder produced it. */
typedef struct {
    int64_t tensor;   /* index into the descriptor */
    int64_t start;    /* first element of the chunk within the tensor */
    int64_t len;      /* number of elements, 1..chunk_elems */
    int32_t dtype;    /* opt2s_dtype of the tensor */
    int32_t reserved;
} opt2s_testing_chunk;

/*
 * Host only (no CUDA call): validate `desc` for `algo` exactly as
 * opt2s_plan_create does and write its chunk list (in launch order) to `out`
 * (capacity `cap` records; `out` may be NULL to query the count).
 * chunk_elems <= 0 selects the library default.  *out_count receives the
 * number of chunks.  Returns OPT2S_OK, a validation error, or
 * OPT2S_ERR_INVALID_ARG when cap is too small.
 */
int opt2s_testing_build_chunks(const TensorListDesc *desc, int32_t algo,
                               int64_t chunk_elems, opt2s_testing_chunk *out,
                               int64_t cap, int64_t *out_count);

/* Host only: the validation opt2s_step performs before any CUDA call. */
int opt2s_testing_validate(const TensorListDesc *desc, const Hyper *hyper,
                           int step);

/* Test build only.  Chunk length (elements, a positive multiple of 8) for
 * plans created afterwards; 0 restores the per-plan choice.  Returns the
 * previous value. */
int64_t opt2s_testing_set_chunk_elems(int64_t chunk_elems);

/* Test build only.  Threads per block (a multiple of 32 in [32, 1024]) and a
 * cap on blocks per launch (>= 1) for later launches; 0 restores each default.  A step whose
 * forced width exceeds opt2s_testing_max_block_threads() for its kernel
 * returns OPT2S_ERR_INVALID_ARG without launching. */
int opt2s_testing_set_launch(int block_threads, int max_blocks);

/* Widest block (threads) the step kernel for (algo, skip_zeros) can launch
 * with on the current device (its register use limits it), or a negative
 * opt2s_status. */
int opt2s_testing_max_block_threads(int32_t algo, int32_t skip_zeros);

/* The library's largest chunk length in elements (chunk_elems <= 0 in
 * opt2s_testing_build_chunks means this length). */
int64_t opt2s_testing_default_chunk_elems(void);

/* Host only: the chunk length a plan for `desc` gets on a device with
 * `resident_warps` resident warps of the step kernel: the power of two c in
 * [128, 2048] minimizing ceil(chunks / resident_warps) * (c / 32 + 8), the
 * modelled time of the slowest warp; ties go to the longer chunk.  A
 * collection with a non-empty 16-bit tensor takes 128 only when its chunks
 * fit in one wave (chunks <= resident_warps). */
int64_t opt2s_testing_choose_chunk_elems(const TensorListDesc *desc, int64_t resident_warps);

/* Host only: the tables the bounded-update-norm step (opt2s_step_max_unorm)
 * builds for `desc` when the plan's chunks have `chunk_elems` elements (<= 0:
 * the largest chunk length).  counts[0] = norm blocks (2,048 elements each,
 * per tensor), counts[1] = groups, counts[2] = chunks.  Each non-null array
 * receives, in descriptor order: group_ranges, 2 per group (first block, end
 * block; a group is up to 64 consecutive blocks of one tensor); first_group,
 * count + 1 entries (tensor t owns groups [first_group[t],
 * first_group[t + 1])); chunk_tensor, the tensor of each chunk.  Call with
 * null arrays first to size them.  Validates `desc` like opt2s_step. */
int opt2s_testing_unorm_tables(const TensorListDesc *desc, int32_t algo, int64_t chunk_elems,
                               uint32_t *group_ranges, uint32_t *first_group,
                               uint32_t *chunk_tensor, int64_t *counts);

/* Test build only.  Runs the kernels' exact division by a constant in
 * [2^-25, 1] (the binary64 route for every x, and the fp32 route for the x in
 * its range) and the IEEE division __fdiv_rn side by side on the current
 * device: mode 0, `n` seeded random pairs with x of every class; mode 1, `n`
 * pairs with x/d next to a binary32 rounding boundary; mode 2, `n` seeded
 * divisors (n <= 2^20), each with all 2^32 binary32 x.  Writes how many
 * results differ (NaN equals NaN) to *mismatches.  Synchronous; allocates a
 * counter on the device. */
int opt2s_testing_check_division(uint64_t seed, int64_t n, int32_t mode, int64_t *mismatches);

/* Test build only.  Fault injection on the host: the next `count` device
 * allocations of plan creation fail as if the device were out of memory
 * (OPT2S_ERR_NO_MEMORY). */
int opt2s_testing_fail_allocs(int count);

/* Host only: the quantization tables the 8-bit step uploads with every plan
 * (the signed and unsigned maps, then the slice entries; the layout is
 * described in the library's internal header): `cap` >= 10,496 words.
 * Lets the tests check the library's tables against the oracle's map. */
int opt2s_testing_quant_tables(uint32_t *out, int64_t cap);

/* Number of kernels this library has launched in this process. */
int64_t opt2s_testing_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* OPT2S_TESTING_H */
