/*
 * mla_decode.h -- C ABI of the B200 (sm_100a) Multi-head Latent Attention
 * decode library (libmla_decode.so).
 *
 * The operation.  MLA decode is the running example, ablation subject and
 * headline kernel of "TileLang: Bridging Programmability and Performance in
 * Modern Neural Kernels" (papernotes.org summary: section "一个完整示例：FlashMLA
 * 的两阶段优化" describes it as a first GEMM S = Q K^T with Q and the KV tile in
 * shared memory, a softmax over S, and a second GEMM of the cast scores with
 * V; the main-results table "主实验", row FlashMLA, and the hackmd essay
 * "TileLang 完整解析", section "FlashMLA Benchmark", time it).  The pages leave
 * the formula to the reader; this library computes the textbook definition:
 * for every sequence b, query token t < Sq and head h < H, with L = seqlens[b],
 *
 *     s_j          = softmax_scale * sum_{d<576} q[b,t,h,d] * kv[b,j,d]    (j < L)
 *     out[b,t,h,e] = sum_j exp(s_j - max s) kv[b,j,e] / sum_j exp(s_j - max s)  (e < 512)
 *     lse[b,t,h]   = ln sum_j exp(s_j)                          (natural log)
 *
 * i.e. many query heads attend over ONE shared compressed latent cache whose
 * rows are 576 wide (512 latent + 64 rope); the values are the first 512
 * columns of the same rows.  The Sq query tokens of a sequence all see keys
 * 0..L-1 (no mask between them).  L = 0 gives out = 0 and lse = -inf.
 *
 * Numerics: bf16 inputs, fp32 accumulation in the tensor cores, fp32 online
 * softmax in base 2 (as in the online-softmax fragment of "DeepSeekV4-
 * TileLang", qingkeai.online, section "TileLang 的设计精髓"), bf16 output.
 *
 * Conventions for every entry point:
 *   - The caller owns all memory.  The library never allocates device memory;
 *     it keeps no global state besides a per-process cache of the CUDA driver
 *     entry point it uses to encode TMA descriptors.
 *   - Pointers named "device" must be device pointers of the plan's device;
 *     "host" pointers are ordinary host memory.
 *   - Work is enqueued on `stream` and runs asynchronously; a return of MLA_OK
 *     means the arguments were valid and the launches were accepted.  Faults
 *     detected on the device (timeouts, lengths out of range) are recorded in
 *     the workspace and reported by mla_decode_check().
 *   - No entry point throws, aborts or prints.
 */
#ifndef MLA_DECODE_H_
#define MLA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mla_status {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,   /* a null pointer, a size out of range, an inconsistent plan */
    MLA_ERR_ALIGNMENT = 2,     /* a pointer not 16-byte aligned (TMA needs 16-byte aligned bases) */
    MLA_ERR_UNSUPPORTED = 3,   /* a shape this build has no kernel for (see mla_decode_plan) */
    MLA_ERR_CUDA = 4,          /* a CUDA runtime / driver call failed (launch, attribute, ...) */
    MLA_ERR_TIMEOUT = 5,       /* device: a bounded pipeline wait ran out; results are invalid */
    MLA_ERR_WORKSPACE = 6,     /* workspace pointer null or smaller than the plan requires */
    MLA_ERR_SEQLEN = 7         /* device: some seqlens[b] was < 0 or > L_max (clamped to [0, L_max]) */
} mla_status;

/* Kernel variants a plan can select. */
enum {
    MLA_KERNEL_TRANSPOSED = 1, /* S^T = K Q^T per CTA, kv rows on the 128 TMEM lanes (any H*Sq) */
    MLA_KERNEL_PAIR = 2,       /* CTA pair, 64 query rows per CTA, cta_group::2 MMAs (H*Sq % 128 == 0) */
    MLA_KERNEL_MHA = 3,        /* MHA decode (mha_decode_plan): the transposed kernel over 128-wide K, V */
    MLA_KERNEL_FP8 = 4,        /* MLA decode over an FP8 cache (mla_decode_plan_fp8): the transposed kernel
                                  with E4M3 chunks widened to f16 in shared memory */
    MLA_KERNEL_FP8_MMA = 5,    /* MLA decode over an FP8 cache with the codes as kind::f8f6f4 MMA operands
                                  (what mla_decode_plan_fp8 picks; see mla_decode_plan_fp8_kernel) */
    MLA_KERNEL_FP8_PAIR = 6    /* MLA decode over an FP8 cache on a CTA pair: the pair kernel's dataflow with
                                  the codes as kind::f8f6f4 operands (H*Sq % 128 == 0) */
};

/*
 * Launch plan.  Filled by mla_decode_plan(); treat as read-only.  Plain data:
 * it may be copied, kept for any number of runs and freed by the caller.
 */
typedef struct mla_plan {
    int32_t B, Sq, H, L_max;   /* problem shape the plan was made for */
    int32_t device;            /* CUDA device ordinal */
    int32_t num_sms;           /* multiprocessors on that device */
    int32_t kernel;            /* MLA_KERNEL_* */
    int32_t group_rows;        /* query rows (token, head pairs) handled per CTA */
    int32_t num_groups;        /* CTAs (or CTA pairs) that share one KV partition */
    int32_t num_partitions;    /* KV partitions: the flattened KV tiles of all sequences are cut into
                                  this many balanced contiguous ranges */
    int32_t tile_kv;           /* kv rows per pipeline tile */
    int32_t cta_threads;       /* threads per CTA of the main kernel */
    uint64_t smem_bytes;       /* dynamic shared memory per CTA of the main kernel */
    uint64_t workspace_bytes;  /* bytes the caller must provide to mla_decode_run */
    int32_t l2_prefetch_tiles; /* KV tiles the loader prefetches into L2 ahead of its shared-memory
                                  loads (0..16; a tuning knob, does not change results) */
    int32_t split_tiles;       /* 0: balanced split-KV schedule (where a sequence is cut depends on the
                                  whole batch); > 0: batch-invariant schedule, every sequence cut into
                                  chunks of this many tiles (mla_decode_plan_batch_invariant) */
    int32_t Hkv;               /* kv heads: 1 for MLA (one latent cache); MHA: query head h reads kv head
                                  h / (H / Hkv) */
    int32_t head_dim;          /* width of a key row: 576 (MLA), 128 (MHA) */
    uint64_t reserved[4];
} mla_plan;

/*
 * mla_decode_plan -- validate a shape and choose kernel, grid and workspace.
 *
 *   B          number of sequences, 1 <= B <= 65535
 *   Sq         query tokens per sequence, 1 <= Sq <= 16
 *   H          query heads, one of 16, 32, 64, 128
 *   L_max      rows allocated per sequence in kv, 1 <= L_max <= 2^24
 *   device     CUDA device ordinal (must be an sm_100 device at run time)
 *   num_partitions_override
 *              0 = automatic (balanced over the device's SMs); > 0 forces that
 *              many KV partitions (tests use it to force 1 = no split, or
 *              many splits); it is clamped to [1, 4096]
 *   plan       (host, out) filled on success
 *   workspace_bytes
 *              (host, out, may be NULL) size of the device workspace to pass
 *              to mla_decode_run; the workspace is caller-owned, must be
 *              256-byte aligned, and must be zeroed once (mla_decode_workspace_init)
 *              before its first use
 *
 * Returns MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED or MLA_ERR_CUDA
 * (device query failed).  Does not launch anything.
 */
mla_status mla_decode_plan(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                           int32_t num_partitions_override, mla_plan* plan, size_t* workspace_bytes);

/*
 * mla_decode_plan_kernel -- mla_decode_plan with an explicit kernel choice:
 * kernel = 0 (automatic: MLA_KERNEL_PAIR when Sq*H is a multiple of 128, else
 * MLA_KERNEL_TRANSPOSED), MLA_KERNEL_TRANSPOSED (any supported shape) or
 * MLA_KERNEL_PAIR (MLA_ERR_UNSUPPORTED unless Sq*H % 128 == 0).  Both kernels
 * compute the same result; the choice only changes speed.  Other arguments,
 * outputs and return codes as for mla_decode_plan.
 */
mla_status mla_decode_plan_kernel(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                                  int32_t num_partitions_override, int32_t kernel, mla_plan* plan,
                                  size_t* workspace_bytes);

/*
 * mla_decode_plan_batch_invariant -- a plan whose results do not depend on
 * the rest of the batch: a sequence's out and lse are bitwise the same
 * whatever other sequences (and how many) share the call.  The qingkeai.online
 * essay on TileLang in the DeepSeek-V4 report (section "V4 设计报告里的几个点",
 * its third point on precision and bitwise alignment) stresses batch
 * invariance of kernels for uses such as RL; it gives no schedule, and this
 * is one.  The balanced schedule of mla_decode_plan cuts the flattened KV
 * tiles of the whole batch into equal ranges, so where a sequence is cut (and
 * hence the rounding of its partials and their merge) depends on the other
 * sequences.  Here every sequence is cut into chunks of split_tiles KV tiles
 * (128 keys each; its last chunk shorter) at fixed offsets from its start;
 * each chunk is processed on its own and the chunks are merged in order, so
 * only the placement of work on the GPU depends on the batch.
 *
 *   split_tiles  tiles per chunk, 1 <= split_tiles <= 131072; 0 = 16 (2048
 *                keys).  Sequences of at most split_tiles tiles are computed
 *                whole.  Smaller chunks spread one long sequence over more
 *                SMs; larger ones write fewer partials.
 * Other arguments and return codes as mla_decode_plan (no partition
 * override: the partition count only places chunks).  The workspace holds one
 * partial per chunk of B sequences of L_max keys.  Run with mla_decode_run,
 * mla_decode_run_sinks or mla_decode_run_noalloc (if the workspace fits its
 * scratch).  For a given split_tiles, kernel choice depends only on Sq * H.
 */
mla_status mla_decode_plan_batch_invariant(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                                           int32_t split_tiles, mla_plan* plan, size_t* workspace_bytes);

/*
 * mla_decode_workspace_init -- zero the workspace's status words on `stream`
 * (asynchronous cudaMemsetAsync of the header).  Call once per workspace before
 * the first run; mla_decode_check() re-zeroes them after reading.
 */
mla_status mla_decode_workspace_init(const mla_plan* plan, void* workspace, size_t workspace_bytes,
                                     void* stream);

/*
 * mla_decode_run -- enqueue one MLA decode on `stream` (a cudaStream_t; NULL =
 * the legacy default stream).
 *
 *   q         device, bf16 [B, Sq, H, 576], contiguous row-major, 16-byte aligned
 *   kv        device, bf16 [B, L_max, 576], contiguous; values are kv[..., :512]
 *   seqlens   device, int32 [B], 0 <= seqlens[b] <= L_max (rows >= seqlens[b]
 *             are never read; out-of-range values are clamped and flagged)
 *   softmax_scale  multiplies q.k (576^-0.5 for MLA)
 *   out       device, bf16 [B, Sq, H, 512], contiguous, 16-byte aligned (written)
 *   lse       device, fp32 [B, Sq, H] (written; natural-log log-sum-exp of the
 *             scaled scores, -inf for an empty sequence)
 *   workspace device, workspace_bytes >= plan->workspace_bytes, 256-byte aligned;
 *             holds split-KV partial outputs and the status words.  A workspace
 *             must not be used by two runs that may execute concurrently.
 *
 * Launches the main kernel and the split-KV combine kernel; no host sync, no
 * allocation, so the call can be captured in a CUDA graph.
 * Returns MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_WORKSPACE,
 * MLA_ERR_UNSUPPORTED (device is not sm_100) or MLA_ERR_CUDA.
 */
mla_status mla_decode_run(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                          float softmax_scale, void* out, float* lse, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * mla_decode_run_phase -- the two launches of mla_decode_run, one at a time:
 * phase 1 = the main kernel (partials and finished sequences), phase 2 = the
 * split-KV combine kernel (merges partials, writes empty sequences).  Issuing
 * phase 1 then phase 2 on one stream is exactly mla_decode_run; separate calls
 * let a caller place events or other work between them.  Same arguments and
 * return codes as mla_decode_run, plus MLA_ERR_INVALID_ARG for another phase.
 */
mla_status mla_decode_run_phase(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                                float softmax_scale, void* out, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream, int32_t phase);

/*
 * mla_decode_run_sinks -- mla_decode_run with attention sinks: one extra
 * logit per head that enters every row's softmax denominator and carries no
 * value.  "TileLang: Bridging Programmability and Performance in Modern
 * Neural Kernels" (papernotes.org summary) lists an attention-sink kernel in
 * its main-results table (section "主实验", row "Attention Sinks") and notes
 * in "关键发现" that it differs from standard attention by a few lines; the
 * formula is not printed, and this is its plain reading.  For a row of head h
 * with scaled scores s_j (j < L) and sink logit sigma_h:
 *     m = max(sigma_h, max_j s_j),   l = sum_j exp(s_j - m) + exp(sigma_h - m)
 *     out = sum_j exp(s_j - m) v_j / l,   lse = m + ln l   (natural log)
 * An empty sequence gives out = 0 and lse = sigma_h.
 *
 *   sinks     device, fp32 [H], 4-byte aligned, in the units of the scaled
 *             scores (it is not multiplied by softmax_scale); the same logits
 *             apply to every sequence and query token.  NULL = no sinks
 *             (exactly mla_decode_run); -inf entries switch one head's sink off.
 * Every other argument, the launches and the return codes are those of
 * mla_decode_run.
 */
mla_status mla_decode_run_sinks(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                                float softmax_scale, const float* sinks, void* out, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * mla_decode_check -- synchronize `stream`, read and clear the workspace's
 * device status words.  Returns MLA_OK if no run since the last check
 * recorded a fault, else MLA_ERR_TIMEOUT / MLA_ERR_SEQLEN (the first recorded),
 * or MLA_ERR_CUDA if the synchronization itself failed.
 */
mla_status mla_decode_check(const mla_plan* plan, void* workspace, void* stream);

/*
 * mla_decode_run_noalloc -- mla_decode_run without a caller workspace.  The
 * decode papers have no counterpart to this call; it exists for callers that
 * must not allocate device memory while decoding: a serving engine that hands
 * almost all HBM to its KV cache at start-up and cannot spare a workspace
 * later, or a plain C host that has no device allocator to draw from.
 *
 * The split-KV partials and the status words live in one static device array
 * of MLA_NOALLOC_SCRATCH_BYTES inside this library.  Every GPU that loads the
 * library holds that array until the process exits; the call itself allocates
 * nothing (no cudaMalloc, no cudaFree, no allocating library routine).
 *
 *   plan, q, kv, seqlens, softmax_scale, out, lse, stream
 *             as for mla_decode_run; inputs and outputs are still the
 *             caller's device buffers
 *   wait_and_check
 *             0: only enqueue, like mla_decode_run; device-recorded faults are
 *             then not reported (the next call clears them).
 *             non-zero: also synchronize `stream` and read the status words,
 *             returning MLA_ERR_TIMEOUT or MLA_ERR_SEQLEN like mla_decode_check
 *
 * The first call on a device looks up the array's device address there (with
 * that device current), which may load the library's device code onto it:
 * make that first call outside any stream capture.  Each call clears the
 * status words on `stream` before its launches; the partial slots keep the
 * previous call's contents, which nothing reads.  All calls on a device share
 * the one array, so two calls whose work can overlap on the GPU (different
 * streams without ordering, several host threads) race and give wrong
 * results: order them on one stream.
 *
 * Returns the codes of mla_decode_run, plus MLA_ERR_WORKSPACE when the plan
 * needs more than MLA_NOALLOC_SCRATCH_BYTES of scratch (every automatic plan
 * for a 148-SM device fits; a large num_partitions_override may not), checked
 * before anything is enqueued, and MLA_ERR_UNSUPPORTED for a device ordinal
 * of 64 or more.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (40u * 1024u * 1024u)
mla_status mla_decode_run_noalloc(const mla_plan* plan, const void* q, const void* kv, const int32_t* seqlens,
                                  float softmax_scale, void* out, float* lse, int32_t wait_and_check,
                                  void* stream);

/*
 * MHA decode -- the second workload on the same skeleton: standard
 * multi-head attention decode with grouped kv heads and separate K and V
 * tensors of width 128.  The TileLang summary lists MHA in its main-results
 * table ("TileLang: Bridging Programmability and Performance in Modern
 * Neural Kernels", papernotes.org, section "主实验", row "MHA"); no formula
 * is printed, and this is the textbook one.  For sequence b, token t, head h,
 * kv head hk = h / (H / Hkv), L = seqlens[b]:
 *     s_j = scale * <q[b,t,h,:], k[b,j,hk,:]>   (j < L)
 *     out[b,t,h,:] = sum_j softmax(s)_j v[b,j,hk,:],   lse = ln sum_j exp(s_j)
 * The Sq tokens of a sequence all see keys 0..L-1.  It runs on the transposed
 * kernel: one CTA per (KV partition, kv head), its columns the Sq * (H / Hkv)
 * query rows that share the kv head, padded to 16 or 32.
 *
 * mha_decode_plan -- as mla_decode_plan, with
 *   H, Hkv     query and kv heads: 1 <= Hkv, H % Hkv == 0, Sq * (H / Hkv) <= 32
 *   B, Sq, L_max, device, num_partitions_override, plan, workspace_bytes
 *              as mla_decode_plan (Sq <= 16)
 * Returns MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED or MLA_ERR_CUDA.
 */
mla_status mha_decode_plan(int32_t B, int32_t Sq, int32_t H, int32_t Hkv, int32_t L_max, int32_t device,
                           int32_t num_partitions_override, mla_plan* plan, size_t* workspace_bytes);

/*
 * mha_decode_run -- enqueue one MHA decode on `stream`.
 *   q       device, bf16 [B, Sq, H, 128], contiguous, 16-byte aligned
 *   k, v    device, bf16 [B, L_max, Hkv, 128] each, contiguous, 16-byte aligned
 *   seqlens device, int32 [B], as for mla_decode_run
 *   softmax_scale  multiplies q.k (128^-0.5 for standard attention)
 *   sinks   device fp32 [H] per-head attention-sink logits (see
 *           mla_decode_run_sinks) or NULL
 *   out     device, bf16 [B, Sq, H, 128] (written);  lse  device, fp32 [B, Sq, H]
 *   workspace  as for mla_decode_run, plan->workspace_bytes
 * Launches the main kernel and the split-KV combine; no host sync, no
 * allocation.  Return codes as mla_decode_run; MLA_ERR_INVALID_ARG for a
 * plan not made by mha_decode_plan.
 */
mla_status mha_decode_run(const mla_plan* plan, const void* q, const void* k, const void* v, const int32_t* seqlens,
                          float softmax_scale, const float* sinks, void* out, float* lse, void* workspace,
                          size_t workspace_bytes, void* stream);

/* mha_decode_run_phase -- the launches of mha_decode_run one at a time (1 =
 * main kernel, 2 = split-KV combine), as mla_decode_run_phase. */
mla_status mha_decode_run_phase(const mla_plan* plan, const void* q, const void* k, const void* v,
                                const int32_t* seqlens, float softmax_scale, const float* sinks, void* out, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream, int32_t phase);

/*
 * FP8 latent cache.  The hackmd essay "TileLang 完整解析" (section "冷靜看待：
 * TileLang 的局限與挑戰") names FP8 as the precision where TileLang trails or
 * fails and prints no format; this library takes the common reading of an
 * FP8 KV cache: every element of the [B, L_max, 576] cache is an OCP E4M3
 * code (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, subnormals
 * at exponent 0, S.1111.111 = NaN, largest finite 448) and
 *     kv_value[b, j, d] = kv_scale * e4m3(kv_fp8[b, j, d])
 * with one fp32 kv_scale for the whole cache.  The decode is the definition
 * at the top of this file on those values (keys: all 576 columns; values:
 * the first 512), with q bf16, out bf16 and lse fp32 as there.
 *
 * Numerics, by kernel (all keep the cache's values exact and accumulate in fp32):
 *   MLA_KERNEL_FP8_PAIR (the default when Sq*H is a multiple of 128): the
 *     codes are the operands of kind::f8f6f4 MMAs on a CTA pair; each q row is
 *     scaled by a power of two and carried as the sum of two E4M3 terms (about
 *     8 significant bits, the precision of a bf16 q), and P (scaled by 2^4) as
 *     the sum of two (about 8 bits, the precision of the bf16 P of the bf16
 *     path).
 *   MLA_KERNEL_FP8_MMA (the default otherwise): the codes are the operands of
 *     kind::f8f6f4 tensor-core MMAs as they are; each q row is scaled by a
 *     power of two and carried as the sum of three E4M3 terms (about 12
 *     significant bits, relative error <= 2^-12), and P (scaled by 2^4) as the
 *     sum of two (about 8 bits, the precision of the bf16 P of the bf16 path).
 *   MLA_KERNEL_FP8: every E4M3 value divided by 2^8 is exact in f16, so the
 *     kernel widens the codes to those f16 values in shared memory (integer
 *     bit moves) and runs f16 x f16 -> f32 MMAs; q is narrowed from bf16 to f16
 *     (exact for 2^-17 <= |q| <= 65504; |q| > 65504 becomes inf, smaller |q|
 *     lose at most 2^-25), P is rounded to f16, and kv_scale * 2^8 multiplies
 *     the scores (with softmax_scale) and the output rows.
 *
 * mla_decode_plan_fp8 -- as mla_decode_plan (same arguments, limits and return
 * codes) for an FP8 cache; the plan's kernel is MLA_KERNEL_FP8_PAIR (128-row
 * query groups on CTA pairs, 256 threads, the bf16 pair plan's partitions) when
 * Sq*H is a multiple of 128, else MLA_KERNEL_FP8_MMA (16 or 32 query rows per
 * CTA, 192 threads).
 */
mla_status mla_decode_plan_fp8(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                               int32_t num_partitions_override, mla_plan* plan, size_t* workspace_bytes);

/*
 * mla_decode_plan_fp8_kernel -- mla_decode_plan_fp8 with an explicit kernel:
 *   kernel  0: what mla_decode_plan_fp8 picks;
 *           MLA_KERNEL_FP8_PAIR: the codes as MMA operands on CTA pairs
 *           (MLA_ERR_UNSUPPORTED unless Sq*H % 128 == 0);
 *           MLA_KERNEL_FP8_MMA: the codes as MMA operands, transposed
 *           orientation, any supported shape;
 *           MLA_KERNEL_FP8: the widening kernel (f16 operands, 320 threads).
 *           Anything else: MLA_ERR_INVALID_ARG.
 * Other arguments and return codes as mla_decode_plan_fp8; the plan runs
 * through mla_decode_run_fp8.
 */
mla_status mla_decode_plan_fp8_kernel(int32_t B, int32_t Sq, int32_t H, int32_t L_max, int32_t device,
                                      int32_t num_partitions_override, int32_t kernel, mla_plan* plan,
                                      size_t* workspace_bytes);

/*
 * mla_decode_run_fp8 -- enqueue one MLA decode over an FP8 cache on `stream`.
 *   plan     from mla_decode_plan_fp8 (any other plan: MLA_ERR_INVALID_ARG)
 *   q        device, bf16 [B, Sq, H, 576], contiguous, 16-byte aligned
 *   kv_fp8   device, E4M3 codes (one byte each) [B, L_max, 576], contiguous,
 *            16-byte aligned; rows at or past seqlens[b] are never used
 *   kv_scale the cache's dequantization scale, finite and > 0
 *            (else MLA_ERR_INVALID_ARG)
 *   seqlens, softmax_scale, out, lse, workspace, workspace_bytes, stream
 *            as mla_decode_run;  sinks as mla_decode_run_sinks (NULL = none)
 * Launches the main kernel and the split-KV combine; no host sync, no
 * allocation; return codes as mla_decode_run.  The cache must hold finite
 * codes (a quantiser saturates): a NaN code (S.1111.111) in a used row gives
 * unspecified results (NaN with MLA_KERNEL_FP8_MMA, +-480 * kv_scale with
 * MLA_KERNEL_FP8).
 */
mla_status mla_decode_run_fp8(const mla_plan* plan, const void* q, const void* kv_fp8, float kv_scale,
                              const int32_t* seqlens, float softmax_scale, const float* sinks, void* out, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/* mla_decode_run_fp8_phase -- the launches of mla_decode_run_fp8 (no sinks) one
 * at a time (1 = main kernel, 2 = split-KV combine), as mla_decode_run_phase. */
mla_status mla_decode_run_fp8_phase(const mla_plan* plan, const void* q, const void* kv_fp8, float kv_scale,
                                    const int32_t* seqlens, float softmax_scale, void* out, float* lse,
                                    void* workspace, size_t workspace_bytes, void* stream, int32_t phase);

/* Static English description of a status code (never NULL). */
const char* mla_status_string(mla_status status);

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
int32_t mla_decode_abi_version(void);

/*
 * Test hooks (not for production use).  mla_decode_set_debug() sets
 * process-wide options applied to subsequent runs:
 *   wait_timeout_ns  bound of every device pipeline wait (0 = default, 2 s)
 *   stall_tile       >= 0: the TMA producer of the first CTA skips the load of
 *                    that pipeline unit while still arming its barrier, so the
 *                    consumer's bounded wait runs out (exercises the timeout
 *                    path without faulting or hanging the GPU); -1 = off
 */
mla_status mla_decode_set_debug(uint64_t wait_timeout_ns, int32_t stall_tile);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H_ */
