/*
 * mac.h -- C ABI of the MAC-Attention decode step on NVIDIA B200 (sm_100a).
 *
 * MAC-Attention ("MAC-Attention: a Match-Amend-Complete Scheme for Fast and
 * Accurate Attention Computation", page 1, abstract) speeds up long-context
 * decoding by reusing attention already computed for a recent, similar query:
 *   Match    -- the current pre-RoPE query is compared by L2 distance with a
 *               short window of recent queries;
 *   Amend    -- on a hit, the keys of a small band before the matched
 *               query's position are recomputed with the current query;
 *   Complete -- fresh attention over the KV tail is merged with the reused,
 *               amended state by a numerically stable log-sum-exp merge.
 * On a miss the step is ordinary split-KV decode attention over every key.
 * On a hit the work does not grow with the context length.
 *
 * Conventions used by every entry point
 *   - Group: each KV head serves G = num_q_heads / num_kv_heads query heads
 *     (page 1 states that the method works with MQA and GQA): G from 1
 *     (multi-head attention) to 8, or 16, 32 or 64 (multi-query attention
 *     sized groups, e.g. 32 query heads over one KV head); other sizes return
 *     MAC_ERR_SHAPE.  One match decision is taken per (sequence, KV head)
 *     over its G heads.  Groups of 16-64 heads read each K/V row from memory
 *     once for the whole group: at head_dim 128 the group is one tensor-core
 *     tile (tcgen05 products with tensor-memory accumulators, then a merge
 *     launch), at head_dim 64 chunks of 8 heads share every box.  They take
 *     no per-head matching, and every key range runs through partial
 *     results (the whole-unit setting does not apply to them).
 *   - Distance: mean over the G heads of the squared L2 distance between the
 *     pre-RoPE queries.  Hit iff the smallest distance over the window is
 *     strictly below tau; ties go to the more recent entry; NaN never hits.
 *     Only entries whose position precedes the current one are candidates.
 *   - Window: the W most recent previous decode steps of the same sequence
 *     (per KV head).  The first step after init or reset always misses.
 *   - Cut: every step stores (pre-RoPE query, prefix state over keys
 *     [0, c_t), position p_t) with c_t = max(0, p_t - band).  A hit on an
 *     entry at position p_s reuses its prefix state over [0, c_s),
 *     c_s = max(0, p_s - band), recomputes [c_s, c_t) (amend) and [c_t, p_t]
 *     (complete) with the current query.  A miss computes [0, c_t) and
 *     [c_t, p_t].
 *   - RoPE: K in the cache is post-RoPE.  The library rotates q_pre to
 *     rope_pos with rotate-half pairs (i, i + D/2), inv_freq_i =
 *     rope_theta^(-2i/D), angles in fp64.  Scores are q.k / sqrt(D).
 *   - Positions: step attends keys [0, seq_lens[b] - 1]; p_t = seq_lens[b]-1.
 *     The step's own K/V row must already be in the cache (see
 *     mac_append_kv).
 *   - Memory: every tensor argument is caller-owned.  "device" pointers are
 *     CUDA device memory of the device that was current at mac_init_state;
 *     "host" pointers are host memory (pinned for overlap, pageable works).
 *     The library owns only its MacState (ring buffers and scratch).
 *   - Streams: `stream` is a cudaStream_t (NULL = legacy default stream).
 *     Device entry points only enqueue work and never synchronise; calls on
 *     one MacState must be ordered on one stream.
 *   - Errors: every int-returning function returns MAC_OK or a MAC_ERR_*
 *     code; host-side validation failures enqueue nothing.  Faults found on
 *     the device (bad sequence length, bad page id, a wait that timed out)
 *     set bits of a device status word, write NaN to the affected unit's out
 *     and lse and leave its window unchanged; mac_get_status reads them.
 */
#ifndef MAC_B200_H
#define MAC_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    MAC_OK = 0,
    MAC_ERR_ARG = 1,    /* NULL where a pointer is required, misaligned pointer, value out of range */
    MAC_ERR_SHAPE = 2,  /* unsupported head_dim / group size / page size / window */
    MAC_ERR_CUDA = 3,   /* a CUDA runtime or driver call failed */
    MAC_ERR_OOM = 4,    /* device allocation failed */
    MAC_ERR_DEVICE = 5  /* the device status word is non-zero (see mac_get_status) */
};

/* Bits of the device status word. */
#define MAC_DEV_BAD_SEQ_LEN 1u /* seq_lens[b] < 1 or beyond the cache capacity */
#define MAC_DEV_BAD_PAGE 2u    /* a block-table entry needed by the step is outside [0, num_pages) */
#define MAC_DEV_TIMEOUT 4u     /* a bounded wait inside a kernel gave up; outputs of that launch are invalid */

typedef struct MacConfig {
    int batch;             /* B >= 1 */
    int num_q_heads;       /* Hq */
    int num_kv_heads;      /* Hkv; Hq must be a multiple of it, Hq / Hkv in 1..8, 16, 32 or 64 */
    int head_dim;          /* D: 64 or 128 */
    int window;            /* W: entries kept per (sequence, KV head), 1..256 */
    int band;              /* b >= 0: keys before the match position that are recomputed */
    float tau;             /* match threshold on the mean squared L2 distance (strict <); 0 = never hit */
    double rope_theta;     /* RoPE base (> 0) */
    int page_size;         /* 0: contiguous K/V [B][max_seq][Hkv][D]; else tokens per page, a multiple of 16 */
    int max_seq;           /* contiguous: rows per sequence in K/V (capacity); paged: unused */
    int max_pages_per_seq; /* paged: row length of block_table; capacity = max_pages_per_seq * page_size */
    int num_pages;         /* paged: pages P in the K/V pools [P][page_size][Hkv][D] */
    int cut_mode;          /* where a stored prefix ends, c = max(0, p - band + cut_mode):
                            * 0 (default) the band is the b keys before the match position,
                            * 1 it ends at the match position itself; other values MAC_ERR_ARG */
    int match_per_head;    /* 0 (default): one match decision per (sequence, KV head) over its G
                            * query heads; 1: one decision per query head (its own squared L2
                            * distance, nearest entry and reuse boundary), the KV head then reads
                            * the union of its heads' key ranges once; hit_mask and match_pos
                            * become [B][Hq].  Other values MAC_ERR_ARG; groups of more than 8
                            * heads MAC_ERR_SHAPE.  (Page 1: the method composes with MQA/GQA;
                            * the page does not fix the granularity.) */
    int q_bf16;            /* 0 (default): q_pre is fp32; 1: q_pre holds bf16 bit patterns (uint16) */
    int ring_bf16;         /* 0 (default): the window keeps fp32 queries and outputs; 1: it keeps
                            * them as bf16 (round to nearest even from fp32; m and l stay fp32),
                            * halving the window scan and state bytes of a hit */
} MacConfig;

typedef struct MacState MacState; /* opaque; owns device memory on the device current at init */

/* Allocate the ring buffers (queries, (o, m, l) states, positions, step
 * counters) and the scratch of one layer, on the current device.  Every
 * sequence starts with an empty window.  *out receives the new state.
 * Returns MAC_ERR_SHAPE for unsupported shapes, MAC_ERR_OOM / MAC_ERR_CUDA
 * when allocation fails (nothing is leaked).  Synchronous. */
int mac_init_state(const MacConfig *cfg, MacState **out);

/* Release every device buffer of the state.  Waits for the device. */
void mac_destroy(MacState *st);

/* Empty the window of sequence b (all its KV heads): its next step misses.
 * Enqueued on stream. */
int mac_reset_seq(MacState *st, int b, void *stream);

/* One MAC decode step of every sequence and KV head (page 1: match, then
 * amend and complete on a hit, split-KV attention on a miss, stable merge).
 *   q_pre       device [B][Hq][D] pre-RoPE queries, fp32 (bf16 bits with
 *               q_bf16), 16-byte aligned.
 *   rope_pos    device int32 [B], position used to rotate the queries.
 *   K, V        device bf16 bit patterns (uint16), 16-byte aligned:
 *               contiguous [B][max_seq][Hkv][D] or paged [P][page_size][Hkv][D].
 *   block_table device int32 [B][max_pages_per_seq] (paged), NULL if contiguous.
 *   seq_lens    device int32 [B], keys visible at this step (p_t = seq_lens - 1).
 *   out         device fp32 [B][Hq][D], attention output.
 *   lse         device fp32 [B][Hq], natural-log log-sum-exp of the scores
 *               the output combines (reused and fresh).
 *   hit_mask    device uint8 [B][Hkv] ([B][Hq] with match_per_head), 1 where
 *               the match hit; may be NULL.
 *   match_pos   device int32 [B][Hkv] ([B][Hq] with match_per_head), position
 *               of the matched entry or -1; may be NULL.
 * The window of every unit advances by one entry.  Enqueues one kernel (the
 * one-launch step, see mac_set_one_launch) or two, and nothing else (no
 * allocation, no host synchronisation), so the call can be recorded into a
 * CUDA graph -- e.g. one graph per token over all layers' states -- and
 * replayed; the recording holds the K/V addresses it saw.
 * Reproducibility: hit/miss decisions never depend on the work split, but
 * on large steps (at least 4096 keys of work per SM) the split learns each
 * SM's streaming rate from earlier steps by default, so the order in which
 * partial results are merged -- and with it the last bits of out and lse --
 * depends on the state's history and on the GPU.  mac_set_reproducible
 * turns the learning off: the same inputs then give the same bits. */
int mac_decode_step(MacState *st, const void *q_pre, const int *rope_pos, const uint16_t *K,
                    const uint16_t *V, const int *block_table, const int *seq_lens, float *out,
                    float *lse, uint8_t *hit_mask, int *match_pos, void *stream);

/* The two halves of mac_decode_step, for callers that time or overlap them.
 * mac_match runs the match stage, rotates the queries, writes hit_mask /
 * match_pos, records the step's query in the window and plans the key
 * ranges; mac_attend runs amend, complete (or the miss path) and the merge
 * using the plan of the preceding mac_match on the same state.  Arguments as
 * in mac_decode_step; mac_match writes NaN to out/lse of invalid units. */
int mac_match(MacState *st, const void *q_pre, const int *rope_pos, const int *block_table,
              const int *seq_lens, float *out, float *lse, uint8_t *hit_mask, int *match_pos,
              void *stream);
int mac_attend(MacState *st, const uint16_t *K, const uint16_t *V, const int *block_table,
               float *out, float *lse, void *stream);

/* Write the step's own K/V rows into the cache at position seq_lens[b] - 1
 * of every sequence (paged-KV manager composition, page 1).
 *   K, V        device bf16 cache, layout as in mac_decode_step (written).
 *   block_table device int32 (paged) or NULL.
 *   seq_lens    device int32 [B].
 *   k_new, v_new device bf16 [B][Hkv][D].
 * Rows whose position or page id is invalid are skipped and flagged in the
 * status word. */
int mac_append_kv(MacState *st, uint16_t *K, uint16_t *V, const int *block_table,
                  const int *seq_lens, const uint16_t *k_new, const uint16_t *v_new, void *stream);

/* Seed every sequence's window from its last n prefill positions (0 <= n <=
 * window), so that the first decode steps can already hit.  Each window is
 * emptied, then position j (oldest first) is stored as a decode step at that
 * position would store it: its pre-RoPE query and its prefix state over keys
 * [0, c), c = max(0, p - band + cut_mode), computed here from the cache with
 * the query rotated at rope_pos (the window of recent queries on the
 * MAC-Attention page, filled before decoding instead of by the first W
 * decode steps).  Cost: n dense passes over each prefix.
 *   q_pre     device [n][B][Hq][D] pre-RoPE queries of the positions (fp32, or
 *             bf16 bits with q_bf16).
 *   rope_pos  device int32 [n][B].
 *   K, V, block_table  the cache, as in mac_decode_step; keys [0, p] of every
 *             position must be in it.
 *   seq_lens  device int32 [n][B]: p + 1 of each position.
 * Enqueued on stream; uses the state's scratch (do not overlap with
 * mac_decode_step_host on the same state).  MAC_ERR_ARG for n outside
 * [0, window] or missing pointers. */
int mac_warm_start(MacState *st, int n, const void *q_pre, const int *rope_pos, const uint16_t *K,
                   const uint16_t *V, const int *block_table, const int *seq_lens, void *stream);

/* mac_append_kv (when k_new_h is not NULL) and mac_decode_step with the
 * per-step inputs and outputs in HOST memory: copies q_pre_h, rope_pos_h,
 * seq_lens_h and the new rows to library staging buffers, runs the step,
 * copies out_h, lse_h, hit_h and match_pos_h back (any of the four may be
 * NULL) and synchronises the stream before returning.  K, V, block_table
 * stay device-resident (the cache is state, not a per-step input).  Returns
 * MAC_ERR_DEVICE if the device status word is non-zero after the step.
 * The inputs go through one pinned host block and one copy each way; the
 * copy-in, append, step and copy-out are recorded once as a CUDA graph per
 * (K, V, block_table, append or not) and replayed on `stream` by later calls
 * (the work-split setters drop the recording).  Not thread-safe on one
 * state; do not call it while `stream` is being captured. */
int mac_decode_step_host(MacState *st, const void *q_pre_h, const int *rope_pos_h,
                         const int *seq_lens_h, const uint16_t *k_new_h, const uint16_t *v_new_h,
                         uint16_t *K, uint16_t *V, const int *block_table, float *out_h,
                         float *lse_h, uint8_t *hit_h, int *match_pos_h, void *stream);

/* Synchronise the device, copy the status word to *device_status (may be
 * NULL) and clear it.  Returns MAC_ERR_DEVICE if it was non-zero. */
int mac_get_status(MacState *st, int *device_status);

/* Ring state export/import (checkpoint / resume).  The byte layout is:
 * int32 header[8] = {magic 0x4D414331, B*Hkv, W+1, G, D, ring_bf16, 0, 0},
 * then q[U][W+1][G][D] and o[U][W+1][G][D] (fp32, or bf16 bits when
 * ring_bf16; o is the normalised output of each stored prefix state),
 * fp32 m[U][W+1][G] (max score, natural-log units),
 * fp32 l[U][W+1][G] (sum of exp(score - m)), int32 pos[U][W+1],
 * int32 steps[U] (decode steps since reset; entry of step n sits in slot
 * n mod (W+1)).  Both calls synchronise the device.  host_buf must hold
 * mac_state_bytes(st) bytes. */
size_t mac_state_bytes(const MacState *st);
int mac_export_state(const MacState *st, void *host_buf, size_t bytes);
int mac_import_state(MacState *st, const void *host_buf, size_t bytes);

/* Tuning of the work split of the attention kernel.  The key ranges of all
 * units are laid end to end in a cost space where every non-empty range also
 * weighs a fixed per-piece cost (in keys; default 1024) and the space is
 * split evenly over min(grid, ceil(total / min_keys)) CTAs (min_keys default
 * 128).  A larger piece cost spreads many short (hit) ranges over more CTAs
 * when a batch also holds long (miss) ranges. */
int mac_set_min_keys_per_cta(MacState *st, int keys);
int mac_set_piece_cost(MacState *st, int keys);

/* Tuning: a (sequence, KV head) whose fresh key range (amend band + tail on
 * a hit, every key on a miss) holds at most `keys` keys (default 1024) is
 * done end to end by one CTA, with no partial results; longer ranges are
 * cut over several CTAs and merged by the last of them.  0 cuts every
 * range. */
int mac_set_whole_unit_keys(MacState *st, int keys);

/* One-launch step.  For groups of up to 8 query heads per KV head with one
 * decision per KV head (no per-head matching), and at most two units per SM,
 * mac_decode_step runs the whole step as one cooperative launch of one CTA
 * per SM: each CTA matches its own units and finishes every unit with at
 * most whole_unit_keys fresh keys (every hit) on the spot; the last CTA to
 * finish matching lays out the longer ranges (the misses) over all SMs, each
 * SM's range shortened by the whole units it already carries, and the CTAs
 * then stream them.  A hit step then costs one launch and no serial layout.
 * on = 1 (default): use it where the configuration allows; 0: two launches
 * (mac_match, then mac_attend), as every other configuration runs.  Both
 * give the same decisions; outputs agree within rounding.  MAC_ERR_ARG for
 * a NULL state or another value. */
int mac_set_one_launch(MacState *st, int on);

/* 1 if mac_decode_step on this state runs as one launch, else 0. */
int mac_one_launch(const MacState *st);

/* Observability.  With on = 1 every step records, for each CTA of its
 * launch, the %globaltimer time (ns) at which the CTA passed each phase:
 * 0 kernel start, 1 its first unit's query and window loaded, 2 that unit's
 * decision taken, 3 its units matched, 4 its plans published, 5 its first
 * K/V box on chip, 6 the last box of its whole units consumed, 7 its whole
 * units done, 8 the split table published (the laying-out CTA of the
 * one-launch step), 9 the split table seen, 10 its split range done, 11 end
 * (phases 1-2 also in the match kernel of two launches); and adds to
 * four counters: 0 keys attended with the current query (the fresh keys of
 * every unit), 1 pieces walked, 2 units done whole, 3 split units merged.
 * The keys counter checks on the device that a hit reads only its band and
 * tail whatever the context length (page 1: the cost of a hit does not grow
 * with the context).  Costs one small memset per step and a few atomics per
 * piece; 0 (default) turns it off.  MAC_ERR_ARG for a NULL state or another
 * value. */
int mac_set_trace(MacState *st, int on);

/* Copy the last traced step's phase times to stamps ([mac_attend_grid(st)][12]
 * unsigned 64-bit ns; a phase a CTA did not reach is 0; may be NULL, else
 * n_stamps must be at least grid * 12) and the counters accumulated since the
 * last call to counters ([4]; may be NULL), then clear the counters.
 * Synchronises the device. */
int mac_get_trace(MacState *st, unsigned long long *stamps, size_t n_stamps, unsigned long long *counters);

/* Reproducible work split.  on = 1: every step splits the key ranges evenly
 * over the CTAs and no streaming rate is learned or used, so a step's out and
 * lse depend only on its inputs and the window (bit for bit, on any B200);
 * on = 0 (default): large steps size each SM's range by its learned rate
 * (faster all-miss steps, history-dependent rounding).  MAC_ERR_ARG for a
 * NULL state or another value. */
int mac_set_reproducible(MacState *st, int on);

/* Persistent grid size of the attention kernel (CTAs). */
int mac_attend_grid(const MacState *st);

/* Dense split-KV decode attention with no allocation at all.  The paper has
 * no counterpart: this is a convenience for callers that cannot call
 * cudaMalloc -- inference-server plugins and embedded hosts that must take
 * every byte of device memory from their host framework's pre-planned pool
 * or a budget fixed at model load, and latency-critical paths that cannot
 * afford an allocation's implicit device synchronisation.  It computes, for
 * every sequence and KV head, attention of the RoPE'd query group over ALL
 * keys [0, seq_lens[b] - 1] (the miss path of mac_decode_step: no window,
 * no reuse, no MacState) with the same kernels, and keeps all their scratch
 * (about 2 MiB) in one static device array inside the library.
 *   q_pre, rope_pos, K, V, block_table, seq_lens, out, lse: as in
 *       mac_decode_step (device pointers, caller-owned, 16-byte aligned
 *       q_pre, K, V).
 *   device_status: device uint32 receiving MAC_DEV_* bits (OR-ed in, not
 *       cleared); required (NULL returns MAC_ERR_ARG), since it is the only
 *       way a bad sequence length or page id reaches the caller.
 *   batch .. num_pages: shapes as in MacConfig.
 * Limits: batch * num_kv_heads <= 64, batch * num_q_heads <= 256, head_dim
 * 64 or 128, Hq / Hkv an integer from 1 to 8; other shapes return
 * MAC_ERR_SHAPE before anything is enqueued.
 * Nothing is allocated or freed; the static array exists on every device
 * that loads the library until the process exits.  The first call on a
 * device looks up the array's device address and sets kernel attributes
 * (make that first call before any stream capture); a call whose
 * rope_theta or head_dim differs from the previous call's uploads 512 bytes
 * of inverse frequencies from host memory, which cannot happen inside a
 * stream capture: such a call on a capturing stream returns MAC_ERR_ARG
 * (make the first call with new frequencies outside the capture).  Every call shares the one array
 * and finds it as the previous call left it; the call clears the counters
 * that must start at zero.  Two calls whose kernels overlap on the GPU (on
 * different streams, or on the same device from different threads without
 * ordering) race on the array and produce garbage: order them. */
int mac_dense_decode_static(const float *q_pre, const int *rope_pos, const uint16_t *K,
                            const uint16_t *V, const int *block_table, const int *seq_lens,
                            float *out, float *lse, unsigned *device_status, int batch,
                            int num_q_heads, int num_kv_heads, int head_dim, double rope_theta,
                            int page_size, int max_seq, int max_pages_per_seq, int num_pages,
                            void *stream);

/* Self-test of the device-side failure path.  Every wait inside the
 * library's kernels is bounded (2 s of %globaltimer); when one gives up, the
 * kernel sets MAC_DEV_TIMEOUT in its status word, lets its own copies land
 * and returns, so the context stays usable and the host learns of it from
 * the status.  This call enqueues one small kernel that waits, through the
 * same bounded wait, on a barrier nothing arrives on: after about 2 s it
 * ORs MAC_DEV_TIMEOUT into *device_status (device uint32, caller-owned) and
 * exits.  No fault, trap or hang is involved.  Returns MAC_ERR_ARG for a
 * NULL status, MAC_ERR_CUDA if the launch fails. */
int mac_selftest_wait_timeout(unsigned *device_status, void *stream);

/* Static description of a return code. */
const char *mac_error_string(int code);

#ifdef __cplusplus
}
#endif
#endif /* MAC_B200_H */
