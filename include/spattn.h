/*
 * spattn — exact block-sparse softmax attention (forward and backward) for
 * token layouts whose logical blocks are only partly occupied, on NVIDIA
 * B200 (sm_100a).
 *
 * Problem statement: the KPage abstract ("KPage: block-sparse attention for
 * partially occupied 3D blocks", zhuanzhiai.com, abstract paragraph).  A
 * sparse graph over logical blocks of a 3D video token layout decides which
 * query tokens may attend which key tokens; edge blocks of the T x H x W
 * latent grid hold padded rows.  The method packs valid 16-row K/V pages
 * into large tiles while loading, keeps exact per-row masking, and owns the
 * K/V side in the backward pass so the sparse graph is preserved exactly in
 * forward and backward.
 *
 * Data model
 *   - A slot is one row of Q (or K/V).  q_group[i] >= 0 is the query group of
 *     slot i; -1 marks a padded slot that is never a query.  kv_group[j] is
 *     the same for keys.
 *   - The graph is a CSR over (head, query group): entries
 *     kv_groups[row_ptr[r] .. row_ptr[r+1]) with r = head * n_q_groups + a
 *     are the key groups that query group a may attend in that head.  The
 *     same graph serves every batch index, unless layout.graph_batches =
 *     batch: then row r = (b * heads + head) * n_q_groups + a holds batch
 *     entry b's graph.  Duplicate entries are allowed.
 *   - Query slot i may attend key slot j in head h iff both are valid and
 *     kv_group[j] is listed for q_group[i].
 *   - A page is 16 consecutive slots; a Q block is 64 consecutive query
 *     slots.
 *
 * Tensors (all device pointers, owned by the caller)
 *   Q, O, dO, dQ : bf16 [batch, heads, q_slots, head_dim], contiguous
 *   K, V, dK, dV : bf16 [batch, kv_heads, kv_slots, head_dim], contiguous
 *                  (dK, dV of a K/V head sum the gradients of all query
 *                  heads that read it)
 *   LSE          : fp32 [batch, heads, q_slots], natural log of
 *                  sum_j exp(scale * q_i . k_j) over the allowed keys.
 *   Every pointer must be 16-byte aligned.  head_dim is 64 or 128.
 *   Padded input rows may hold any finite values; outputs on padded or
 *   attention-free query rows are O = 0, LSE = -inf, dQ = 0, and on padded
 *   key rows dK = dV = 0.
 *
 * Errors: every call returns an SPATTN_* status; nothing throws across the
 * ABI.  fwd/bwd are asynchronous on `stream` (a cudaStream_t, NULL = the
 * legacy default stream) and launch nothing when an argument is rejected.
 * Kernels never trap: a device-side wait that exceeds its deadline records an
 * error in the plan, which spattn_check() reports.  A plan must not be used
 * by two streams at the same time (the backward workspace is per plan).
 */
#ifndef SPATTN_H_
#define SPATTN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum spattn_status {
  SPATTN_OK = 0,
  SPATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad group id */
  SPATTN_ERR_UNSUPPORTED = 2, /* head_dim not 64/128, slots beyond int32 rows, ... */
  SPATTN_ERR_OOM = 3,         /* spattn_plan ran out of host or device memory (or host threads) */
  SPATTN_ERR_CUDA = 4,        /* a CUDA runtime call failed */
  SPATTN_ERR_TIMEOUT = 5,     /* a kernel gave up on a device-side wait */
  SPATTN_ERR_DEVICE = 6       /* a kernel rejected its work item */
};

typedef struct spattn_plan_s* spattn_plan_t; /* opaque, owned by the library */

typedef struct {
  int32_t batch, heads, head_dim; /* head_dim in {64, 128} */
  int64_t q_slots, kv_slots;      /* >= 1 each; any length (ragged tails allowed) */
  const int32_t* q_group;         /* host [q_slots], -1 = padded */
  const int32_t* kv_group;        /* host [kv_slots], -1 = padded */
  int32_t n_q_groups, n_kv_groups;
  float scale;                    /* softmax scale > 0; 0 selects 1/sqrt(head_dim) */
  int32_t kv_heads;               /* K/V heads for grouped-query attention: heads % kv_heads == 0,
                                     query head h reads K/V head h / (heads / kv_heads);
                                     0 selects kv_heads = heads (1 = multi-query) */
  int32_t graph_batches;          /* 0 or 1: one graph for every batch entry; batch: one graph per
                                     batch entry (the graph then has batch * heads * n_q_groups rows,
                                     batch-major) */
} spattn_layout;

typedef struct {
  const int64_t* row_ptr;   /* host [heads * n_q_groups + 1], non-decreasing, row_ptr[0] = 0 */
  const int32_t* kv_groups; /* host [row_ptr[heads * n_q_groups]], values in [0, n_kv_groups) */
} spattn_graph;

typedef struct {
  int64_t useful_pairs;          /* allowed (query slot, key slot) pairs, all batches and heads */
  int64_t physical_pairs_fwd;    /* pairs computed by the forward tiles (128 rows x 16 per page) */
  int64_t physical_pairs_dkdv;   /* pairs computed by the dK/dV tiles */
  int64_t physical_pairs_dq;     /* pairs computed by the dQ tiles */
  int64_t bsa_pairs;             /* 64x64 x number of (Q block, K block) pairs with any allowed pair */
  int64_t n_work_fwd;            /* forward / dQ work items (all batches) */
  int64_t n_work_dkdv;           /* dK/dV work items (all batches) */
  int64_t n_entries_fwd;         /* (work item, K page) entries of one batch */
  int64_t n_entries_dkdv;        /* (work item, Q page) entries of one batch */
  int64_t device_bytes;          /* device memory held by the plan */
  int64_t launches_fwd;          /* kernels one spattn_fwd call launches */
  int64_t launches_bwd;          /* kernels one spattn_bwd call launches */
  double plan_ms;                /* host time spent in spattn_plan */
} spattn_stats;

/* Kernel ids of spattn_kernel_times. */
enum spattn_kernel {
  SPATTN_K_FWD = 0,   /* forward attention (O, LSE) */
  SPATTN_K_FILL = 1,  /* zero fill of pages without a valid slot */
  SPATTN_K_DELTA = 2, /* rowsum(dO * O) */
  SPATTN_K_DKDV = 3,  /* key-owned dK, dV */
  SPATTN_K_DQ = 4     /* query-owned dQ */
};

typedef struct {
  double ms[5];        /* device time per kernel id, summed over recorded launches */
  int64_t launches[5]; /* recorded launches per kernel id */
} spattn_kernel_times;

/* Build a plan: validate layout and graph, find valid 16-row pages, pack
 * owned tiles, and build the per-tile page lists and masks for the forward /
 * dQ pass (query-owned) and the dK/dV pass (key-owned).
 * Source: the KPage abstract (zhuanzhiai.com paper page), which packs
 * 16-row K/V pages holding valid rows into large tiles across logical-block
 * boundaries, chooses tile shapes for query blocks so that less query-side
 * padding is computed, and has the K/V side own its pages in the backward
 * pass.  Host arrays are
 * copied and may be freed afterwards.  Device lists are allocated on the
 * current device with cudaMalloc and owned by the plan.  On a machine with no
 * usable CUDA device the plan is built on the host only: the inspection
 * calls (stats, pages, qblocks, work) work and spattn_fwd / spattn_bwd /
 * spattn_check return SPATTN_ERR_CUDA. */
int spattn_plan(const spattn_layout* layout, const spattn_graph* graph, spattn_plan_t* out);
/* (Heads are planned in parallel on all hardware threads; the environment
 * variable SPATTN_PLAN_THREADS, if set to n >= 1, uses n threads instead.
 * Heads whose graph rows are identical are planned once and copied
 * (SPATTN_PLAN_DEDUP=0 plans every head; the result is the same).
 * The plan is identical for every thread count.  Per head and pass, the
 * planner groups 64-slot blocks into owned tiles in two ways, slot order and
 * grouping by the overlap of the blocks' column lists, and keeps the one
 * that computes fewer physical pairs; SPATTN_PLAN_PACK=slot or =similar
 * forces one of them.  The query-owned pass may instead take the 64-row
 * route (work word 28, see spattn_plan_work) where a cost model of the
 * forward and dQ steps favours it; SPATTN_PLAN_PACK=route64 forces it.
 * Work items of a head run longest column list first.) */

/* Re-plan for a new sparse graph over the plan's layout, on the GPU.
 * Dynamic block selection (VSA-style graphs, one of the layouts the KPage
 * abstract evaluates, zhuanzhiai.com paper page) changes the graph every
 * call, and host planning of a large graph takes about a second; this call
 * rebuilds both work lists on the device in milliseconds.  row_ptr
 * ([graph_batches * heads * n_q_groups + 1]) and kv_groups ([nnz]) are
 * DEVICE arrays in the format of spattn_graph (rows may be unsorted and hold
 * duplicates), read on `stream`; the plan keeps its own copy.  Grouped-query
 * attention and per-batch graphs are handled as spattn_plan handles them
 * (key-owned entries carry their query-head offset).  The owned tiles are the layout's
 * slot-order tiles (with strided pages); the column lists, strided entries,
 * pair counts and the transposed (key-owned) lists follow the new graph and
 * are identical to what spattn_plan would build with SPATTN_PLAN_PACK=slot,
 * up to the order of the work items.  The call synchronises `stream` once;
 * the new lists are used by every later spattn_fwd / spattn_bwd.  Returns
 * SPATTN_ERR_INVALID_ARG for a malformed graph (the plan is left unchanged),
 * SPATTN_ERR_UNSUPPORTED if one work item would gather more than 8192
 * (head, page, group) triples or a side has 2^24 pages or more,
 * SPATTN_ERR_OOM if growing the plan's device lists
 * fails.  The inspection calls (stats, pages, qblocks, work) describe the
 * new graph (their first call copies it back to the host). */
int spattn_plan_set_graph_device(spattn_plan_t plan, const int64_t* row_ptr, const int32_t* kv_groups, int64_t nnz,
                                 void* stream);

/* Forward: O and LSE for every query slot of every (batch, head): masked
 * softmax attention over exactly the plan's sparse graph, computed over the
 * packed pages; the KPage abstract (zhuanzhiai.com paper page) states that
 * exact masking keeps the original graph intact in the forward pass. */
int spattn_fwd(const void* q, const void* k, const void* v, spattn_plan_t plan, void* o, float* lse,
               void* stream);

/* FP8 (E4M3) quantisation of Q or K for spattn_fwd_fp8: x is a DEVICE bf16
 * tensor [bh, rows, head_dim] (head_dim 64 or 128, 16-byte aligned), read
 * as bh slices (one per batch*head).  Per slice, amax = max |x|; x8
 * (DEVICE, [bh, rows, head_dim] one-byte E4M3 codes: 1 sign, 4 exponent bits
 * with bias 7, 3 mantissa bits, largest finite 448) receives
 * e4m3(x * (448 / amax)) rounded to nearest-even and saturated to +-448, and
 * descale (DEVICE, [bh] fp32, 4-byte aligned) receives amax / 448 (1 for an
 * all-zero slice); every step is one correctly rounded fp32 operation.
 * Inputs must be finite.  Asynchronous on `stream` (four launches).  This
 * is the quantised Q / K line of work that the KPage page lists next to the
 * method (zhuanzhiai.com paper page), applied to the forward only. */
int spattn_quantize_fp8(const void* x, int64_t bh, int64_t rows, int head_dim, void* x8, float* descale,
                        void* stream);

/* Forward with E4M3 Q and K (head_dim 128 only, else
 * SPATTN_ERR_UNSUPPORTED): q8 [batch, heads, q_slots, 128] and k8
 * [batch, kv_heads, kv_slots, 128] hold E4M3 codes, q_descale [batch*heads]
 * and k_descale [batch*kv_heads] their per-slice scales (as written by
 * spattn_quantize_fp8), v is bf16.  Computes exactly what spattn_fwd
 * computes for the dequantised inputs q8 * q_descale and k8 * k_descale: S
 * is a kind::f8f6f4 tensor-core product accumulated in fp32; P, V and O stay
 * bf16 as in spattn_fwd, and LSE is that of the dequantised scores.  Same
 * layouts, alignment, fill of rows without work and error codes as
 * spattn_fwd. */
int spattn_fwd_fp8(const void* q8, const void* k8, const float* q_descale, const float* k_descale, const void* v,
                   spattn_plan_t plan, void* o, float* lse, void* stream);

/* Backward: dQ, dK, dV given O and LSE from spattn_fwd and the loss
 * gradient dO.  Uses the plan's fp32 workspace for rowsum(dO * O) and the
 * plan's work-item counter of the persistent dK/dV kernel, so backward calls
 * on one plan must be ordered (one stream, or events between streams).
 * dK and dV are accumulated per owned key tile and written once, with no
 * atomics: the KPage abstract (zhuanzhiai.com paper page) keeps the graph
 * exact in the backward pass by letting the K/V side own its pages.  The
 * gradient formulas are those of softmax attention. */
int spattn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* d_o,
               spattn_plan_t plan, void* dq, void* dk, void* dv, void* stream);

/* Backward pass that allocates nothing, for callers that cannot allocate
 * device memory when they run it (for example when another allocator has
 * reserved the GPU, or under a fixed device-memory budget).  The paper has
 * no counterpart; it is a deployment variant of spattn_bwd with the same
 * arguments and results.  Its fp32 scratch (one value per query row) is a
 * fixed static device array of 4,194,304 floats (16 MiB) that every GPU
 * loading the library holds until exit, so batch * heads * q_slots must not
 * exceed 4,194,304 (else SPATTN_ERR_UNSUPPORTED, nothing launched).  Each
 * call looks up the array's device address in the current context (no
 * allocation; a device reset therefore cannot leave a stale address), and
 * the first call on each device also loads the library's device code there,
 * so that first call should come before any stream capture.  All
 * calls share the array and every call rewrites what it reads, so calls that
 * overlap on the GPU (on different streams) race with each other. */
int spattn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* d_o, spattn_plan_t plan, void* dq, void* dk, void* dv, void* stream);

/* Synchronise `stream` and report (then clear) any device-side error the
 * plan's kernels recorded: SPATTN_OK, SPATTN_ERR_TIMEOUT or SPATTN_ERR_DEVICE.
 * (Failure reporting; the paper has no counterpart.) */
int spattn_check(spattn_plan_t plan, void* stream);

/* Failure-path self-test of the device-side bounded waits (no fault, no
 * hang).  Launches on `stream` one CTA that waits on a barrier nothing ever
 * completes: one warp with a deadline of `deadline_cycles` SM cycles (10^4 ..
 * 2*10^9, else SPATTN_ERR_INVALID_ARG), one with the tile kernels' deadline.
 * The first times out and records a timeout in the plan's error word, the
 * second sees the CTA's abort flag; both return, and the context stays
 * usable.  The next spattn_check on the plan returns SPATTN_ERR_TIMEOUT (and
 * clears it).  A host-only plan returns SPATTN_ERR_CUDA. */
int spattn_wait_selftest(spattn_plan_t plan, int64_t deadline_cycles, void* stream);

/* Pair accounting of the plan: useful pairs (allowed query-key pairs) and
 * the physical pairs each pass computes, the two counts the KPage abstract
 * (zhuanzhiai.com paper page) compares for its aggregate result, plus the
 * 64x64 block count of a BSA-style kernel for reference.  Fills *stats;
 * never launches. */
int spattn_plan_stats(spattn_plan_t plan, spattn_stats* stats);

/* Per-kernel device timing, for kernel-only measurements like the forward
 * kernel timings the KPage abstract reports (zhuanzhiai.com paper page).  While enabled, spattn_fwd / spattn_bwd record a
 * CUDA event pair around every kernel they launch, on the launch stream.
 * spattn_profile(plan, 1) starts recording, (plan, 0) stops; both discard
 * what was recorded.  spattn_profile_read waits for the recorded events,
 * returns their summed durations and clears the record. */
int spattn_profile(spattn_plan_t plan, int enable);
int spattn_profile_read(spattn_plan_t plan, spattn_kernel_times* out);

/* In spattn_plan_pages and spattn_plan_qblocks, `head` is a graph head:
 * b * heads + h when each batch entry has its own graph, else h. */
/* Canonical page list of (head, Q block): ascending pages holding at least
 * one key that some query of the block may attend (the 16-row K/V pages a Q
 * block needs; KPage abstract, zhuanzhiai.com paper page).  *pages points into a
 * plan-owned buffer that stays valid until the next call on this plan. */
int spattn_plan_pages(spattn_plan_t plan, int32_t head, int64_t qblock, const int32_t** pages, int64_t* n);

/* Transposed list of (head, page): ascending Q blocks whose canonical list
 * holds the page (what a key-owned backward tile walks; KPage abstract,
 * zhuanzhiai.com paper page).  Same buffer rules as spattn_plan_pages. */
int spattn_plan_qblocks(spattn_plan_t plan, int32_t head, int64_t page, const int32_t** qblocks, int64_t* n);

/* Host copy of a work list, for inspection and tests (the packed tiles of
 * the KPage abstract's load-time packing, zhuanzhiai.com paper page).  which = 0: query-owned
 * (forward and dQ), 1: key-owned (dK/dV).  Each work item is 32 int32 words:
 *   [0] batch*heads + head of the owned side (query heads for which = 0,
 *       K/V heads for which = 1)   [1] owned page count n (<= 8)
 *   [2] first entry          [3] end entry (into pages/masks)
 *   [4..11] owned page references   [12..27] 128 row codes, 4 bits each,
 *   row r in word 12 + r/8 at bit 4*(r%8): 0..7 = segment, 14 = owned row
 *   with no segment (padded), 15 = row not written by this item.
 *   [28] route of a query-owned item: 0 = all 128 rows run over the whole
 *   list (entries in ascending slot order); 1 = 64-row route (the KPage
 *   abstract's routing of Q blocks to smaller tiles): rows 0..63 (owned
 *   pages 0..3) and rows 64..127 (owned pages 4..7) each have their own list,
 *   interleaved two entries at a time (entries 4i, 4i+1 for rows 0..63,
 *   4i+2, 4i+3 for rows 64..127, each half ascending; padding entries have
 *   zero masks), so the entry count is a multiple of 4.  [29..31] zero.
 * A page reference p >= 0 is the page of slots 16p .. 16p+15; a negative
 * value is a strided page with base slot b = ~value, whose row r is slot
 * b + 16 (r / 4) + r % 4.  pages[e] is a page reference of the other side;
 * masks[2e] and masks[2e+1] hold eight 16-bit row masks over that page, one
 * per segment (segment s in bits 16 (s % 4) .. 16 (s % 4) + 15 of word
 * masks[2e + s / 4]).
 * Entries are shared by all batch indices. */
int spattn_plan_work(spattn_plan_t plan, int32_t which, const int32_t** work, int64_t* n_work,
                     const int32_t** pages, const uint64_t** masks, int64_t* n_entries);

/* Per entry of work list `which` (as in spattn_plan_work): the query head of
 * the entry relative to the first query head of the item's K/V head (always
 * 0 for the query-owned list and without grouped-query attention); the
 * array has the same length and buffer rules as spattn_plan_work's. */
int spattn_plan_entry_heads(spattn_plan_t plan, int32_t which, const uint16_t** heads, int64_t* n_entries);

/* Free the plan and its device lists (NULL is a no-op).  The caller must
 * make sure no kernel launched with the plan is still running.  (Plan
 * lifetime; the paper has no counterpart.) */
void spattn_plan_destroy(spattn_plan_t plan);

/* Static English text of a status code; never NULL.  (Error reporting; the
 * paper has no counterpart.) */
const char* spattn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SPATTN_H_ */
