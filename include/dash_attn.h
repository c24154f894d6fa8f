/*
 * dash_attn.h -- C ABI of the deterministic attention backward for B200.
 *
 * The library computes the FlashAttention-style backward pass of softmax
 * attention (dQ, dK, dV from Q, K, V, O, dO and the row log-sum-exp) with a
 * persistent sm_100a kernel.  Each CTA runs whole KV-tile chains with dK/dV
 * resident in tensor memory; dQ is accumulated in fp32 through per-block
 * integer tickets so that the partials of every dQ block are added in the
 * fixed order that the chosen schedule defines.  With the same shape, mask,
 * schedule and SM count, results are bitwise identical from run to run.
 *
 * Sources (cited by page title and section):
 *   "Resumen Técnico: DASH – Programación de Atención Determinista para el
 *    Entrenamiento de LLM de Alto Rendimiento" (the DASH technical summary):
 *   §1   deterministic backward = fixed dQ accumulation order; the serialised
 *        baseline and its nondeterministic counterpart
 *   §2.1 the DAG model: compute and reduction phases, accumulation-order
 *        edges, critical path objective, one KV tile per SM as a chain
 *   §2.2.A descending Q-tile iteration; §2.2.B shift scheduling (full masks),
 *        symmetric shift (causal masks) and the zero-weight-edge lemma
 *   §5   the choice between heuristic and optimal schedules is left to the user
 * The pages print no interface and no formulas: the signatures below and the
 * attention definitions are this library's own.
 *
 * Conventions for every GPU entry point:
 *   - Tensors are caller-owned DEVICE memory on the current CUDA device.
 *     q, k, v, o, dout, dq, dk, dv: bf16, contiguous [B, H, S, D], 16-byte
 *     aligned.  lse: fp32 [B, H, S], natural log of sum_j exp(scale * q.k_j).
 *     The softmax scale is 1/sqrt(D).  Causal masks are top-left aligned:
 *     query i attends to keys j <= i.
 *   - Supported shapes: D in {64, 128}, S a positive multiple of 128,
 *     B * H * S < 2^31, and a schedule table of at most 2^31 - 1 pairs
 *     (B * H * N^2 for a full mask, half that plus the diagonal for a causal
 *     one, N = S / 128).  Other shapes return DASH_ERR_UNSUPPORTED.
 *   - No C++ exception leaves the library: every entry point returns a status.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous: DASH_OK means the work was enqueued.  Argument and launch
 *     errors are returned at once; errors found on the device (a spin wait
 *     that ran out) are reported by dash_attn_sync_status().
 *   - The library owns its workspace (fp32 dQ accumulators, tickets, the
 *     per-row LSE and Delta terms, an error word) and caches it per
 *     (device, stream); schedule tables are cached per shape.  Calls on
 *     different streams use different workspaces.  Workspace memory is
 *     released by dash_release_workspace().
 */
#ifndef DASH_ATTN_H_
#define DASH_ATTN_H_

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DASH_SCHED_NAIVE_ASC = 0,   /* §1 baseline: Q ascending, dQ order ascending KV       */
  DASH_SCHED_DESCENDING = 1,  /* §2.2.A: Q tiles last to first, dQ order ascending KV  */
  DASH_SCHED_SHIFT = 2,       /* §2.2.B full masks: cyclic shift, conflict-free order  */
  DASH_SCHED_SYM_SHIFT = 3,   /* §2.2.B causal masks: KV i and N-1-i folded, 2 phases  */
  DASH_SCHED_ATOMIC = 4,      /* §1 nondeterministic counterpart: fp32 atomic dQ adds  */
  DASH_SCHED_SHIFT_PAIRS = 5, /* full masks, even N: CTA pairs pre-sum dQ (see below)  */
  DASH_SCHED_SYM_SHIFT_PAIRS = 6 /* causal masks, N % 4 == 0: the same CTA pairs      */
} dash_schedule_t;

typedef enum {
  DASH_OK = 0,
  DASH_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad enum, negative size   */
  DASH_ERR_UNSUPPORTED = 2,   /* shape or schedule/mask combination not provided       */
  DASH_ERR_CUDA = 3,          /* a CUDA runtime call failed                            */
  DASH_ERR_TIMEOUT = 4,       /* a device spin wait ran out (see dash_attn_sync_status)*/
  DASH_ERR_OOM = 5,           /* a device or host allocation failed                    */
  DASH_ERR_SCHEDULE = 6       /* schedule table failed validation (e.g. would deadlock)*/
} dash_status_t;

/*
 * Forward pass, provided only to produce O and LSE for the backward.
 * o: bf16 [B,H,S,D] output.  lse: fp32 [B,H,S] output (natural log).
 * Computes O = softmax(scale * Q K^T + mask) V with fp32 accumulation.
 */
int dash_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                  int B, int H, int S, int D, int causal, void* stream);

/*
 * Backward pass (DASH summary §1, §2.1, §2.2).
 * Inputs q, k, v, o, dout (bf16 [B,H,S,D]) and lse (fp32 [B,H,S]); outputs
 * dq, dk, dv (bf16 [B,H,S,D]), fully overwritten.
 *   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i.v_j - dO_i.O_i),
 *   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,
 *   with P_ij = exp(scale q_i.k_j - LSE_i) (0 where masked).
 * schedule: a dash_schedule_t.  SHIFT needs causal == 0; SYM_SHIFT needs
 * causal == 1 and an even number of 128-row tiles.  Every schedule except
 * ATOMIC is deterministic: dQ partials are added in fp32 in the schedule's
 * fixed order, then rounded once to bf16.
 */
int dash_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                  const void* dout, const float* lse, void* dq, void* dk, void* dv,
                  int B, int H, int S, int D, int causal, int schedule, void* stream);

/*
 * Grouped-query attention (no counterpart on the pages; their baseline models use
 * it).  H query heads share Hkv key/value heads, H / Hkv query heads per K/V head
 * (a power of two): query head h reads K/V head h / (H / Hkv).
 *   q, o, dout, dq: bf16 [B, H, S, D];  k, v, dk, dv: bf16 [B, Hkv, S, D];
 *   lse: fp32 [B, H, S].
 * dK and dV sum over the K/V head's query heads.  The group of H / Hkv query heads is
 * cut into `split` sub-groups of consecutive heads (a power of two dividing H / Hkv).
 * The schedule table runs the chains that feed one dK/dV tile of one sub-group back
 * to back on one CTA, so the sub-group's sum accumulates in the kernel's fp32
 * accumulators, query heads in order.  With split > 1 each sub-group is a unit of
 * its own (more units for the persistent grid, shorter runs); the sub-groups'
 * fp32 partials of a dK/dV tile are added in sub-group order (sub-group s waits,
 * bounded, for s - 1 under a ticket) and the last one rounds to bf16, so the
 * result stays deterministic.  This uses 2 * B * Hkv * S * D fp32 of scratch.
 * dQ is ordered per query head as for dash_attn_bwd.  Hkv == H is dash_attn_fwd /
 * dash_attn_bwd.
 * dash_attn_bwd_gqa lets the library choose split (the smallest power of two that
 * fills the grid's rounds noticeably better; dash_bwd_gqa_split_for reports it);
 * dash_attn_bwd_gqa_split takes it from the caller, 0 meaning the library's choice.
 * Errors: DASH_ERR_INVALID_ARG if Hkv < 1 or does not divide H, or split is negative,
 * not a power of two or does not divide H / Hkv; DASH_ERR_UNSUPPORTED if H / Hkv is
 * not a power of two; otherwise as dash_attn_fwd / dash_attn_bwd.
 */
int dash_attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int Hkv, int S, int D, int causal, void* stream);
int dash_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                      int H, int Hkv, int S, int D, int causal, int schedule, void* stream);
int dash_attn_bwd_gqa_split(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv,
                            int B, int H, int Hkv, int S, int D, int causal, int schedule,
                            int split, void* stream);
/*
 * The split dash_attn_bwd_gqa uses for B * Hkv K/V heads with `group` query heads
 * each on a grid of num_ctas persistent CTAs (dash_bwd_num_ctas).  Host only: no
 * device call.  Errors: DASH_ERR_INVALID_ARG for a NULL split, num_ctas, B, Hkv or
 * group below 1, group not a power of two or causal not 0/1; DASH_ERR_UNSUPPORTED
 * for a length or schedule the backward refuses.
 */
int dash_bwd_gqa_split_for(int num_ctas, int B, int Hkv, int group, int S, int causal,
                           int schedule, int* split);

/*
 * Synchronises `stream`, then returns and clears the device error word of
 * that stream's workspace: DASH_ERR_TIMEOUT if a ticket or pipeline wait of a
 * previous backward on this stream ran out (its outputs are then invalid),
 * DASH_ERR_CUDA if the stream reported an error, else DASH_OK.
 */
int dash_attn_sync_status(void* stream);

/* Human-readable name of a status code (static storage; never NULL). */
const char* dash_status_string(int status);

/*
 * Upper bound, in microseconds, of every device spin wait of later launches
 * (ticket waits and pipeline waits).  Default 10 s, or the environment
 * variable DASH_SPIN_LIMIT_US when set.  us <= 0 restores the default.
 */
int dash_set_spin_limit_us(long long us);

/*
 * How the deterministic backward adds a dQ partial at a middle position of an
 * accumulation chain (DASH summary §1, the serialised accumulation): 0 (default) picks
 * per launch, 1 always adds in L2 with red once the ticket grants the position, 2
 * always loads, adds on the SM and stores.  The additions and their order are the
 * same, so the results are bitwise the same; mode 0 takes red where it measured faster:
 * the descending and naive ascending schedules from 64 tiles, and at D = 64 tables that
 * run two or more query heads per unit (multi-head tables that interleave heads,
 * dash_set_head_interleave; grouped-query sub-groups of two or more heads).  Applies to later
 * dash_attn_bwd / dash_attn_bwd_gqa / dash_attn_bwd_host calls on every stream
 * (dash_attn_bwd_noalloc always loads and stores).  Other modes: INVALID_ARG.
 */
int dash_set_dq_chain_mode(int mode);
/* Whether a deterministic backward of this schedule, length and head dim, launched
 * now with heads_per_unit query heads per unit of its table (dash_bwd_head_interleave
 * for the multi-head entry points; group / split for the grouped-query ones), adds with
 * red (*red = 1) or loads, adds and stores (*red = 0); 0 for ATOMIC.  Host only.
 * Errors: INVALID_ARG for a NULL red, a bad schedule, D not 64/128, heads_per_unit below
 * 1 or S not a positive multiple of 128. */
int dash_dq_chain_uses_red(int schedule, int S, int D, int heads_per_unit, int* red);

/*
 * Placement of the schedule table's CTA slots on the SMs (the die-aware placement the
 * DASH summary §4 motivates: at 16k with a full mask, shift slows down through remote
 * L2 segments).  By SM id: each CTA reads its SM id at start and runs the slot equal
 * to that id's rank in the grid, so a head's consecutive units run on SMs with
 * consecutive ids.  In launch order: the grid's CTA b runs slot b.  mode 0 (default):
 * by SM id from 128 tiles (S >= 16384), where it measured faster, else in launch
 * order; mode 1: always by SM id; mode 2: always in launch order.  The table fixes
 * every order, so results are bitwise the same in every mode.  Applies to later
 * dash_attn_bwd, dash_attn_bwd_gqa, dash_attn_bwd_host and dash_trace_bwd calls
 * (dash_attn_bwd_noalloc keeps mode 0).  Other modes: INVALID_ARG.
 */
int dash_set_slot_placement(int mode);
/* Whether a backward of length S, launched now, places slots by SM id (*by_smid = 1)
 * or in launch order (0).  Host only.  Errors: INVALID_ARG for a NULL output or S not
 * a positive multiple of 128. */
int dash_slot_placement_by_smid(int S, int* by_smid);

/*
 * Head interleaving of a multi-head backward's schedule table (DASH summary §2.1: the
 * schedule fixes each dQ block's accumulation order, and the table fixes the schedule's
 * placement on the SMs).  With 2 (or 4) heads per unit, each KV segment of a unit of the
 * schedule runs for 2 (or 4) consecutive heads in turn, K/V loaded again for each; the
 * heads' dQ blocks then receive their contributions further apart in the grid's steps.
 * The order of every dQ block is still fixed by the table, so results stay bitwise
 * reproducible, but they may differ in rounding from the uninterleaved table.
 * mode 0 (default): the library picks, 2 for SYM_SHIFT at D = 64 when the units still
 * fill the grid's rounds (measured faster there), else 1; mode 1: never; mode 2 or 4:
 * that many heads per unit whenever it divides B * H, the CTA-pair schedules' half
 * tables included.  Applies to later dash_attn_bwd,
 * dash_attn_bwd_host, dash_attn_bwd_noalloc and dash_trace_bwd calls (the grouped-query
 * entry points have their own grouping).  Other modes: INVALID_ARG.
 */
int dash_set_head_interleave(int mode);
/* Heads per unit a multi-head backward takes under the current mode for n_heads = B*H
 * heads on num_ctas persistent CTAs.  Host only.  Errors: INVALID_ARG for a NULL
 * output, num_ctas or n_heads below 1, D not 64/128, a bad schedule or causal flag, or
 * S not a positive multiple of 128. */
int dash_bwd_head_interleave(int num_ctas, int D, int schedule, int n_heads, int S, int causal,
                             int* heads_per_unit);

/*
 * Failure-detection testing.  mode 1: the next deterministic dash_attn_bwd or
 * dash_attn_bwd_noalloc (any stream) runs with a schedule table in which dQ
 * block (head 0, Q tile 0) never receives its first two partials, so its ticket
 * waits run out; the kernel still ends, with DASH_ERR_TIMEOUT reported by
 * dash_attn_sync_status (dash_attn_noalloc_sync_status for the second) and
 * invalid outputs.  The fault is made on the host; no memory outside the
 * call's buffers is touched.  mode 0 cancels.  Other modes: INVALID_ARG.
 */
int dash_inject_fault(int mode);

/* Number of persistent CTAs the backward uses on `device` for head dim D. */
int dash_bwd_num_ctas(int device, int D, int* num_ctas);

/*
 * Device timing of backward launches.  Between dash_profile_begin() and
 * dash_profile_end(), every dash_attn_bwd records CUDA events on its stream
 * around its kernels.  dash_profile_end() waits for them and returns the
 * summed milliseconds of the main (persistent) kernel, of the auxiliary
 * kernels (Delta preprocess, and the fp32-to-bf16 dQ pass of ATOMIC), and the
 * number of backward calls recorded.  Outputs may be NULL.
 */
int dash_profile_begin(void);
int dash_profile_end(double* main_ms, double* aux_ms, long long* launches);

/*
 * Diagnostic: one synchronous backward (same arguments as dash_attn_bwd) with
 * a %globaltimer trace of every (KV tile, Q tile) pair, for measuring the
 * compute time c and the reduction time r of the DAG model (DASH summary
 * §2.1).  host_trace receives up to `cap` u64 entries laid out
 * [num_ctas][rows_per_cta][16] (unused rows stay 0); events per pair: 0 S^T
 * issued, 1 softmax done (seen by the MMA issuer), 2 tile MMAs issued, 3
 * softmax start, 4 dQ partial ready at the reducers, 5 partial drained from
 * TMEM, 6 ticket granted (0 for the first contributor of each of the block's
 * two accumulation chains), 7 reduction published or dQ written, 8 P^T packed
 * (end of the softmax's first phase), 9 start of its second phase, 10 dS ready,
 * 11 P^T seen by the MMA issuer, 12 the issuer starts waiting for the S^T
 * buffer, 13 load-add-store (or atomic adds) done, 14 the reducers start
 * waiting for the ticket, 15 dP^T issued.
 * Allocates and frees its own trace buffer.
 */
int dash_trace_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int S, int D,
                   int causal, int schedule, void* stream, unsigned long long* host_trace,
                   long long cap, int* num_ctas, int* rows_per_cta);

/* Frees every cached workspace and schedule table of the current device
 * (synchronises the device first). */
int dash_release_workspace(void);

/* ---------------------------------------------------------------------------
 * Backward pass that allocates nothing.
 *
 * The paper has no counterpart to this entry point.  It serves callers that
 * cannot call cudaMalloc: runtimes that hand out all device memory from their
 * own pool and forbid allocations outside it, and embedded or certified
 * deployments that must fix their device footprint before they start.
 *
 * Same arguments, supported shapes, schedules and results as dash_attn_bwd
 * (q..dv caller-owned device memory; the caller still passes every input and
 * output), bit for bit on the deterministic schedules.  All scratch memory comes
 * from one statically allocated device array of DASH_NOALLOC_SCRATCH_BYTES bytes,
 * which every GPU that loads the library holds until the process exits.  The
 * call never calls cudaMalloc, cudaFree or an allocating library routine.
 *   - Size limit: the array must hold the two fp32 dQ accumulators per block
 *     (2*B*H*S*D*4 bytes), 16 bytes of LSE and Delta terms per row (B*H*S*16), two
 *     tickets per 128-row dQ block and the schedule table; larger calls return
 *     DASH_ERR_OOM without touching the device.
 *   - Set-up: the first call on a device (with that device current) looks up
 *     the array's device address and sizes the persistent grid.
 *   - Schedule tables: a call whose (B*H, S, causal, schedule) differs from the
 *     previous call's copies its table from host memory into the array; while
 *     the stream is being captured that copy is refused with
 *     DASH_ERR_UNSUPPORTED.
 *   - Sharing: every call uses the same array, which keeps the previous call's
 *     contents; the call clears what must start at zero.  Calls that overlap
 *     on the GPU (for example on two streams without ordering between them)
 *     race on the array and give wrong results.
 *   - Errors: device-side timeouts of this entry point are recorded in the
 *     array's error word, which dash_attn_noalloc_sync_status reads; the spin
 *     limit is the one dash_set_spin_limit_us sets (else DASH_SPIN_LIMIT_US,
 *     else 10 s).
 */
#define DASH_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int dash_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv,
                          int B, int H, int S, int D, int causal, int schedule, void* stream);

/*
 * Status of dash_attn_bwd_noalloc on the current device: waits for `stream`,
 * then returns and clears the array's error word.  DASH_ERR_TIMEOUT if a
 * device wait ran out in a call since the word was last read (that call's
 * outputs are invalid), DASH_ERR_UNSUPPORTED if a launch refused to run,
 * DASH_OK otherwise (also before the first call on the device); DASH_ERR_CUDA
 * if the stream reports an error.  Allocates nothing.  The paper has no
 * counterpart to this call either.
 */
int dash_attn_noalloc_sync_status(void* stream);

/* ---------------------------------------------------------------------------
 * Backward pass from host buffers.
 *
 * The paper has no counterpart to this entry point; it serves callers whose
 * tensors live in host memory.  Same arguments, shapes, schedules and results
 * as dash_attn_bwd, except that q, k, v, o, dout, lse and dq, dk, dv are HOST
 * pointers (caller-owned, same layouts; page-locked memory lets the copies run
 * asynchronously and overlap the compute, pageable memory works but copies
 * synchronously).  The heads are split into up to 8 parts.  Each part's inputs
 * are copied to the device on a library-owned stream while the previous part
 * computes on `stream` and the part before that is copied back on a second
 * library-owned stream, through two device staging slots.
 *   - Results: every part runs the sub-table of the whole problem's schedule
 *     table that covers its heads (same CTA for every chain, same position for
 *     every dQ partial), so dq, dk, dv are bitwise identical to those of
 *     dash_attn_bwd on device copies of the same inputs.
 *   - Completion: the call returns once everything is queued; the results are
 *     on the host when `stream` has completed (dash_attn_sync_status(stream)
 *     waits for it and reports device-side timeouts as for dash_attn_bwd).
 *   - Ownership: the staging slots (about 2 * (8*D*2 + 4) bytes per row of one
 *     part), the copy streams and the per-part tables are cached per (device,
 *     stream) and freed by dash_release_workspace().  Calls that use the same
 *     stream are ordered; the host buffers must stay valid and unmodified until
 *     `stream` has completed.
 */
int dash_attn_bwd_host(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                       int H, int S, int D, int causal, int schedule, void* stream);

/* ---------------------------------------------------------------------------
 * Host-only entry points (no GPU needed).
 */

/*
 * Schedule table of a whole grid (DASH summary §2.2), in CTA order.
 * n_heads = B*H heads of N = S/128 tiles on num_ctas persistent CTAs
 * (1 <= num_ctas <= 65536; tables of at most 2^31 - 1 pairs).
 * If rows != NULL, writes up to cap rows of 6 ints:
 *   (cta, head, kv_tile, q_tile, position_in_dQ_order, chain_index).
 * Returns the total number of rows (pairs), or a negative dash_status_t
 * (-DASH_ERR_UNSUPPORTED, -DASH_ERR_SCHEDULE if validation fails).
 */
long long dash_sched_table(int n_heads, int N, int causal, int schedule, int num_ctas,
                           int* rows, long long cap);

/*
 * DASH_SCHED_SHIFT_PAIRS.  The pages name 2-CTA pairs as the answer to the register
 * and TMEM pressure of one KV tile per SM (DASH summary §4) and print no schedule for
 * them; this is the library's.  CTAs 2i and 2i + 1 run KV tiles 2m and 2m + 1 of a
 * head over the same Q tiles at the same steps, Q tile m + t mod N at step t, and the
 * two dQ partials of a step are added together before the ordered accumulation, so a
 * dQ block receives N / 2 contributions, in (round, step) order.  Full mask, N even.
 * DASH_SCHED_SYM_SHIFT_PAIRS is the causal counterpart: KV pair m and Q pair j (Q tiles
 * 2j and 2j + 1) form a pair-tile, present when j >= m; the half table runs
 * DASH_SCHED_SYM_SHIFT over the N / 2 pair-tiles, each pair-tile as two steps (Q tile 2j,
 * then 2j + 1).  On a diagonal pair-tile the step (KV 2m + 1, Q 2m) lies wholly above the
 * diagonal: that CTA computes it as zeros, so both CTAs keep the same steps.  A dQ block
 * q receives q / 2 + 1 contributions.  Causal mask, N a multiple of 4.
 * For these schedules dash_sched_table returns the half table, one row per pair of KV
 * tiles (kv = m, num_ctas counting CTA pairs); dash_sched_table_pairs returns the grid's
 * table for num_ctas CTAs (even), SHIFT_PAIRS for causal = 0 and SYM_SHIFT_PAIRS for
 * causal = 1: rows as for dash_sched_table, slot 2i with KV tile 2m and slot 2i + 1 with
 * KV tile 2m + 1, both with the pair's Q tiles and positions.  Returns the number of
 * rows, or -DASH_ERR_INVALID_ARG (odd num_ctas, causal not 0 or 1),
 * -DASH_ERR_UNSUPPORTED or -DASH_ERR_SCHEDULE.
 * The backward runs them through dash_attn_bwd, the pair being a thread-block cluster of
 * two CTAs: each CTA adds the two partials for half of the columns and accumulates that
 * half in order.  At D = 64 each CTA stages its dQ partial in shared memory and reads the
 * peer's; at D = 128 (the partial stays in TMEM) each reducer thread writes the peer's
 * half of its row into a 16 KiB buffer of the peer's shared memory, 32 columns a round.
 * The other mask and unsupported N return DASH_ERR_UNSUPPORTED.  dash_attn_bwd_host takes them too (its parts are slices
 * of the same table, so the bits are dash_attn_bwd's); the grouped-query, no-allocation
 * and trace entry points return DASH_ERR_UNSUPPORTED.
 */
long long dash_sched_table_pairs(int n_heads, int N, int causal, int num_ctas, int* rows,
                                 long long cap);

/*
 * The part of that table covering heads [h0, h1) (0 <= h0 < h1 <= n_heads), as the
 * host-buffer path launches it: heads renumbered from 0, every chain on the same CTA
 * and every pair at the same position in its dQ order as in the whole table.  Rows
 * as for dash_sched_table.  Returns the number of rows, or -DASH_ERR_INVALID_ARG for
 * a bad head range, -DASH_ERR_UNSUPPORTED, or -DASH_ERR_SCHEDULE if the part fails
 * validation.
 */
long long dash_sched_table_part(int n_heads, int N, int causal, int schedule, int num_ctas,
                                int h0, int h1, int* rows, long long cap);

/*
 * The table of a grouped-query backward: n_heads query heads, `group` per K/V head
 * (n_heads a multiple of group).  Rows as for dash_sched_table, heads being query
 * heads; the chains that feed one dK/dV tile (K/V head = head / group, KV tile) are
 * consecutive on one CTA.  group = 1 gives dash_sched_table's table.  Returns the
 * number of rows, or -DASH_ERR_INVALID_ARG, -DASH_ERR_UNSUPPORTED or
 * -DASH_ERR_SCHEDULE.
 */
long long dash_sched_table_gqa(int n_heads, int group, int N, int causal, int schedule,
                               int num_ctas, int* rows, long long cap);

/*
 * DAG simulation of a schedule table (DASH summary §2.1): per pair the events
 * start, partial ready, reduction start, reduction done; arcs of weight
 * w_compute (tile compute) and w_reduce (ordered reduction), zero-weight
 * chain arcs, one reduction at a time per CTA, and with dq_buffers >= 1 at
 * most that many partials in flight per CTA (<= 0: unbounded).  The
 * accumulation order of a dQ block is one fixed chain when dq_chains = 1 (the
 * pages' model); with dq_chains = K > 1 (the kernel uses 2) position p waits
 * for position p - K and the block's last contributor for the last position
 * of every other chain.  Outputs (any may be NULL): critical_path (longest
 * path), makespan (latest end of a compute phase), bubble_time (sum over used
 * CTAs of critical_path minus the CTA's compute time), stalls (pairs whose
 * partial waited for a free buffer).  Returns DASH_ERR_INVALID_ARG for
 * negative weights or dq_chains < 1.
 * Argument mapping for a caller thinking in (B, H, S): n_heads = B * H and
 * N = S / 128, since the table depends on those two alone; dq_chains has no
 * counterpart in a single-order model (pass 1 for the pages' model); a bubble
 * figure splits into bubble_time (idle time) and stalls (a count).
 */
int dash_sched_simulate(int n_heads, int N, int causal, int schedule, int num_ctas,
                        double w_compute, double w_reduce, int dq_buffers, int dq_chains,
                        double* critical_path, double* makespan, double* bubble_time,
                        long long* stalls);

/*
 * The same simulation of the grouped-query table of dash_sched_table_gqa
 * (n_heads query heads, `group` of them per K/V head): each pair's events and
 * arcs as above, over the grouped table's CTA order and dQ positions.
 * DASH_ERR_INVALID_ARG also when group < 1 or does not divide n_heads.
 */
int dash_sched_simulate_gqa(int n_heads, int group, int N, int causal, int schedule,
                            int num_ctas, double w_compute, double w_reduce, int dq_buffers,
                            int dq_chains, double* critical_path, double* makespan,
                            double* bubble_time, long long* stalls);

/*
 * Checks a schedule table supplied by the caller, in the row format of
 * dash_sched_table: n_rows rows of 6 ints (cta, head, kv_tile, q_tile,
 * position, chain_index), grouped by CTA in ascending order, each CTA's rows in
 * execution order, consecutive rows of one chain sharing its chain index.
 * Checks that every pair of the mask appears once, that positions form a
 * permutation per dQ block, that chains are unbroken, and that the ticket
 * order cannot deadlock when all num_ctas CTAs run concurrently (DASH summary
 * §2.1).  rows is read only.  Returns DASH_OK, DASH_ERR_INVALID_ARG for a
 * malformed row list, or DASH_ERR_SCHEDULE when a check fails.
 */
int dash_sched_check(int n_heads, int N, int causal, int num_ctas, const int* rows,
                     long long n_rows);

/*
 * Longest paths of a general DAG with n_nodes nodes and n_edges weighted
 * edges src[e] -> dst[e] (weight w[e]); host arrays.  Writes depth[n] (longest
 * path ending at the node), height[n] (longest path starting there) and *cp
 * (any may be NULL).  Used to check the lemma of DASH summary §2.2.B.
 * Returns DASH_ERR_INVALID_ARG on a cycle or an out-of-range node.
 */
int dash_dag_longest_path(int n_nodes, int n_edges, const int* src, const int* dst,
                          const double* w, double* depth, double* height, double* cp);

#ifdef __cplusplus
}
#endif
#endif /* DASH_ATTN_H_ */
