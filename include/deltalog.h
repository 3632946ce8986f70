/*
 * deltalog.h -- C ABI of the DeltaLog decode library for B200 (sm_100a).
 *
 * DeltaLog ("DeltaLog: Deferred Materialization of Recurrent States for
 * Linear Attention Decoding", Abstract and AI Summary) keeps each head's
 * recurrent state as a dense base plus a bounded log of recent compact
 * updates.  A decode step reads base + log, appends one compact factor
 * instead of writing the whole state back, and a periodic merge folds the
 * log into the base.  The model observes the same dense state as eager
 * decoding (up to floating-point rounding order).
 *
 * Recurrences (state S is d_v x d_k per head, row = value index, contiguous
 * along the key index):
 *   GDN   S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,  o_t = S_t q_t
 *   KDA   S_t = S_{t-1} Diag(a_t) (I - b_t k_t k_t^T) + b_t v_t k_t^T,  o_t = S_t q_t
 *   RWKV6 (stored as the transpose of its d_k x d_v matrix)
 *         S_t = S_{t-1} Diag(w_t) + v_t k_t^T,
 *         o_t = S_{t-1} r_t + (sum_c r_c u_c k_c) v_t
 *   GDN-2 S_t = S_{t-1} Diag(a_t) (I - (e_t o k_t) k_t^T) + (w_t o v_t) k_t^T,
 *         o_t = S_t q_t   (e_t: erase gate per key channel, w_t: write gate
 *         per value row; the log is KDA's, u_t = w_t o v_t - S' (e_t o k_t))
 * With gamma_t the decay accumulated since the base was last merged and
 * u_t = b_t (v_t - a_t S_{t-1} k_t) (GDN; KDA uses S_{t-1}(a_t o k_t)),
 *   S_t = S_b Diag(gamma_t) + sum_i u_i (k_i o gamma_t / gamma_i)^T,
 * so one log entry is (u_i, k_i, log gamma_i); RWKV6 stores u_i = v_i.
 *
 * Conventions for every call:
 *   - Returns DL_OK (0) or a negative DL_ERR_* code.  Arguments are checked
 *     on the host before anything is enqueued; a failed check enqueues
 *     nothing and changes no state.
 *   - Device pointers are plain CUDA device addresses owned by the caller.
 *     The library never allocates device memory and never frees caller
 *     memory; a dl_state borrows the three buffers sized by dl_state_bytes
 *     for its whole life.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on it and never synchronize, except
 *     dl_state_reset and dl_device_error, which say so.
 *   - One dl_state is used from one host thread and one stream at a time.
 *   - Floating-point results equal eager decoding up to rounding order, not
 *     bitwise: the log and the merge sum in a different order.
 */
#ifndef DELTALOG_H
#define DELTALOG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Recurrence family (the DeltaLog page builds it for GDN, KDA and RWKV6), plus
 * GDN-2 (Gated DeltaNet-2 abstract: separate channel-wise erase and write
 * gates; KDA when both are the same scalar). */
enum dl_variant { DL_GDN = 0, DL_KDA = 1, DL_RWKV6 = 2, DL_GDN2 = 3 };

/* Element type of q (r), k and v as stored by the caller. */
enum dl_dtype { DL_F32 = 0, DL_BF16 = 1 };

/* Status codes. */
enum dl_status {
  DL_OK = 0,
  DL_ERR_ARG = -1,         /* null pointer, bad size, bad enum, bad mode   */
  DL_ERR_ALIGN = -2,       /* a pointer violates the alignment rule        */
  DL_ERR_LOG_FULL = -3,    /* a sequence's log holds L entries: merge first */
  DL_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed          */
  DL_ERR_UNSUPPORTED = -5, /* valid but not built (head size, dtype)        */
  DL_ERR_DEVICE = -6       /* a kernel recorded an error (dl_device_error)  */
};

/* dl_merge modes. */
enum dl_merge_mode {
  DL_MERGE_FULL = 0, /* fold the logs of sequences whose log holds L entries */
  DL_MERGE_ALL = 1   /* fold every non-empty log                            */
};

/* dl_config.flags */
enum dl_flags {
  /* The step kernel merges in place: a head whose append would fill its
   * log writes the merged base instead and leaves an empty log, so the log
   * is never full and dl_merge(DL_MERGE_FULL) has nothing to do. */
  DL_FLAG_FUSED_MERGE = 1,
  /* Bit 2 is reserved (DL_ERR_ARG if set). */
  /* Kaczmarz step size (KLA, GDN and KDA only): the `beta` argument of a
   * step carries the gate eta_t and the kernels use
   * beta_t = eta_t / (|k_t|_2^2 + kla_eps) ("Kaczmarz Linear Attention"
   * abstract), so the write projects exactly whatever the key's norm.
   * With kla_eps = 0 a zero key gives an infinite beta_t, and the outputs
   * are NaN exactly as the formula's are: use kla_eps > 0 where keys may
   * vanish.  Not for RWKV6 or GDN-2 (DL_ERR_ARG). */
  DL_FLAG_KLA = 4,
  /* int8 base quantized once per window ("LeapQuant" abstract: the state
   * is quantized only at the end of a window of tokens, and outputs inside
   * the window use the fixed low-bit state plus high-precision buffered
   * updates; here the window is the stretch between two merges of a
   * sequence's log, and the log stays fp32).  The base holds int8 codes
   * and one fp32 scale per value row:
   *   amax_j = max_c |x_jc|,  inv_j = 127 / amax_j,
   *   code_jc = round-half-even(x_jc * inv_j),  scale_j = amax_j / 127,
   * each an fp32 operation rounded once (rows with amax_j < 2^-120 store
   * zero codes and scale 0); the base value is code_jc * scale_j.  Every
   * merge (DL_MERGE_FULL, DL_MERGE_ALL, the fused merge) folds the log in
   * fp32 and requantizes the rows it writes; dl_state_reset and
   * dl_state_load_seqs quantize the states they load. */
  DL_FLAG_BASE_Q8 = 8
};

/* Layer configuration.  d_k, d_v in {64, 128}; 1 <= L <= 64; B, H >= 1 and
 * B*H*d_v*d_k < 2^40.  `flags` is a bitwise OR of dl_flags.  `step_split`
 * is into how many work items (of d_v / step_split rows) the step kernel
 * cuts one head: 0 picks the library's default (2 for GDN at d_v = 128,
 * else 1), otherwise 1, 2 or 4 with
 * d_v / step_split >= 32 (a performance knob only: results do not depend
 * on it). */
typedef struct dl_config {
  int32_t variant;    /* enum dl_variant */
  int32_t B;          /* sequences in the batch */
  int32_t H;          /* heads per sequence */
  int32_t d_k;        /* key (and q / r) size per head */
  int32_t d_v;        /* value size per head */
  int32_t L;          /* log capacity: entries per head before a merge */
  int32_t in_dtype;   /* enum dl_dtype of q/r, k, v */
  int32_t flags;      /* enum dl_flags */
  int32_t step_split; /* 0 (default), 1, 2 or 4 */
  float kla_eps;      /* epsilon of the KLA step size (DL_FLAG_KLA), >= 0 */
} dl_config;

typedef struct dl_state dl_state;

/* Sizes in bytes of the three device buffers a state borrows:
 *   base: fp32 [B, H, d_v, d_k]                 the dense base S_b; with
 *         DL_FLAG_BASE_Q8 int8 codes [B, H, d_v, d_k] followed, at the
 *         next 256-B boundary, by the fp32 row scales [B, H, d_v]
 *   log : per head L entries of u (fp32 [d_v]; in_dtype for RWKV6),
 *         k (in_dtype [d_k]) and log-decay g (fp32, [1] for GDN, [d_k]
 *         otherwise), laid out as three arrays [B,H,L,.], each 256-B aligned
 *   meta: two int32 fill arrays [B, H] (read and written alternately by
 *         successive steps) and a device error word, each 256-B padded.
 * Any output pointer may be NULL.  Errors: DL_ERR_ARG, DL_ERR_UNSUPPORTED. */
int dl_state_bytes(const dl_config* cfg, size_t* base_bytes, size_t* log_bytes,
                   size_t* meta_bytes);

/* Creates a state over caller-owned device buffers of at least the sizes
 * above, each 256-byte aligned (else DL_ERR_ALIGN).  The contents are
 * undefined until dl_state_reset.  Enqueues nothing.  The handle (host
 * memory) is owned by the library until dl_state_destroy. */
int dl_state_create(const dl_config* cfg, void* base, void* log, void* meta,
                    dl_state** out);

/* Loads a dense state and starts every log.  S0: fp32 [B, H, d_v, d_k]
 * device buffer 16-B aligned, or NULL for a zero state (an int8 base
 * stores Q(S0), quantized row by row as described at DL_FLAG_BASE_Q8).  fill0: host int32
 * [B] with 0 <= fill0[b] < L, or NULL for zeros; sequence b starts with
 * fill0[b] log entries that change nothing (u = 0, k = 0, g = 0), so its
 * first merge comes after L - fill0[b] steps (ragged batches sit at
 * different merge phases).  Clears the device error word.  Synchronizes
 * `stream` before returning (it copies the fill counts from host memory). */
int dl_state_reset(dl_state* st, const float* S0, const int32_t* fill0, void* stream);

/* Loads dense states into some sequences and empties their logs, leaving
 * every other sequence untouched: the slot admission of continuous
 * batching (a finished sequence's slot takes a new one).  seqs: host int32
 * [n], distinct, each in [0, B).  S: fp32 [n, H, d_v, d_k] device buffer
 * (16-B aligned; entry i is the state of sequence seqs[i]) or NULL for zero
 * states.  The loaded sequences' fills become 0.  Asynchronous on `stream`.
 * Errors: DL_ERR_ARG (bad or repeated index, n < 0), DL_ERR_ALIGN. */
int dl_state_load_seqs(dl_state* st, int n, const int32_t* seqs, const float* S, void* stream);

/* One decode step for all B*H heads (one kernel launch).  Defines: the
 * DeltaLog page, Abstract -- a decode step reads the base and the log and
 * appends compact update factors instead of writing the full state back.
 *   q: q_t (r_t for RWKV6)  [B, H, d_k] in_dtype
 *   k: k_t                  [B, H, d_k] in_dtype
 *   v: v_t                  [B, H, d_v] in_dtype
 *   decay: fp32, GDN alpha_t [B, H]; KDA and GDN-2 alpha_t [B, H, d_k];
 *          RWKV6 w_t [B, H, d_k]; every value in (0, 1]
 *   beta: fp32 [B, H] for GDN/KDA; GDN-2: the erase gate e_t [B, H, d_k];
 *         ignored (may be NULL) for RWKV6
 *   bonus: fp32 [H, d_k] RWKV6 u; GDN-2: the write gate w_t [B, H, d_v];
 *          ignored (may be NULL) otherwise
 *   o: fp32 [B, H, d_v] output o_t
 * All pointers 16-byte aligned device addresses.  Without
 * DL_FLAG_FUSED_MERGE, returns DL_ERR_LOG_FULL (enqueuing nothing) when
 * some sequence's log already holds L entries: call dl_merge first.
 * The launch carries each sequence's current fill (from the host-side
 * mirror) by value, so a CUDA graph captured around this call would replay
 * the fills of the captured step: do not capture it. */
int dl_decode_step(dl_state* st, const void* q, const void* k, const void* v,
                   const float* decay, const float* beta, const float* bonus,
                   float* o, void* stream);

/* Folds logs into the base: S_b <- S_b Diag(gamma) + sum_i u_i (k_i o
 * gamma / gamma_i)^T, then empties those logs.  Defines: the DeltaLog page,
 * Abstract -- periodic merge steps fold the log back into the dense base.
 * mode DL_MERGE_FULL folds the sequences whose log holds L entries,
 * DL_MERGE_ALL every non-empty log.  Enqueues nothing when no sequence qualifies.  Like
 * dl_decode_step, the launch carries the qualifying sequences and their
 * fills by value (do not capture it in a CUDA graph). */
int dl_merge(dl_state* st, int mode, void* stream);

/* Writes the dense state S_t = base folded with the log to S_out (fp32
 * [B, H, d_v, d_k], 16-B aligned, must not alias the base) without changing
 * the state.  An int8 base is dequantized (code * scale) before the fold.
 * Defines: the DeltaLog page, Abstract -- the model observes the same dense
 * state as in eager decoding; this call produces that state on demand. */
int dl_materialize(const dl_state* st, float* S_out, void* stream);

/* Eager dense step, the comparison point: reads and writes the whole fp32
 * state S [B, H, d_v, d_k] (16-B aligned) in place, same recurrence and
 * arguments as dl_decode_step.  Defines: the DeltaLog page, Abstract --
 * eager decoding writes the full recurrent state back after every token.  cfg->L and every flag but DL_FLAG_KLA are
 * ignored (the state is always fp32). */
int dl_eager_step(const dl_config* cfg, float* S, const void* q, const void* k,
                  const void* v, const float* decay, const float* beta,
                  const float* bonus, float* o, void* stream);

/* Copies the host-side fill counts (entries per sequence, int32 [B]). */
int dl_state_fill(const dl_state* st, int32_t* fill_out);

/* Releases the handle (not the borrowed buffers).  NULL is accepted. */
int dl_state_destroy(dl_state* st);

/* Reads and optionally clears the device error word that kernels set when
 * a bounded wait gives up or a device-side check fails (code 0 = none;
 * *head = first failing head).  Synchronizes `stream`.
 *   - A state has its own word (in its meta buffer).  A nonzero code after a
 *     step or a merge means some head's work was skipped part-way (a step
 *     may already have advanced that head's fill, a merge may have folded
 *     only some rows): the state is invalid until dl_state_reset.
 *   - `st` NULL reads the one word per device that every dl_eager_step call
 *     and dl_selftest_wait_timeout share: the first error recorded wins, so
 *     with overlapping eager calls the head index may belong to either, and
 *     the self-test clears the word (erasing what an earlier eager call
 *     recorded). */
int dl_device_error(dl_state* st, int32_t* code, int32_t* head, int clear, void* stream);

/* Exercises the kernels' failure path on the current device without a
 * fault: one warp waits, with the same bounded wait the kernels use, on a
 * shared-memory barrier nothing completes; after about one second it gives
 * up, records the timeout in the device error word the eager kernel uses
 * and returns.  *code receives the recorded code (1 = wait timed out),
 * read back and cleared.  Synchronizes `stream`. */
int dl_selftest_wait_timeout(int32_t* code, void* stream);

/* Total kernels this library has launched in this process. */
uint64_t dl_launch_count(void);

/* Static text for a status code. */
const char* dl_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* DELTALOG_H */
