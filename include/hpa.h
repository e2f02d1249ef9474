/*
 * hpa.h -- paged mixed-length decode attention for NVIDIA B200 (sm_100a).
 *
 * C ABI of libhpa.so.  One decode step of one attention layer is
 *
 *     hpa_kv_prologue   (optional: RMSNorm + RoPE of the new token's q/k and
 *                        the K/V write into its cache slot)
 *     hpa_decode_plan   (per-step tile plan from the device-side lengths)
 *     hpa_decode_run    (persistent paged GQA decode + log-sum-exp merge)
 *
 * all asynchronous on one CUDA stream, with no host synchronisation in
 * between, so a step can be captured in a CUDA graph.  hpa_decode_step and
 * hpa_decode_step_prologue make the plan inside the decode kernel (two
 * launches per step).  A batch whose sequences' pages are spread over
 * several GPUs is decoded per GPU with hpa_decode_step_lse and the GPUs'
 * states combined with hpa_merge_states.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device (or managed) pointers owned by
 *     the caller; the library never allocates, frees or retains them past the
 *     call.  Host pointers are read or written before the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued on it; the call returns without waiting.
 *   - Arguments are validated on the host before anything is enqueued; a bad
 *     argument returns an error and enqueues nothing.  Values that only the
 *     device sees (lengths, page ids, positions) are checked by the kernels,
 *     which never trap: they skip the offending access and set a bit in a
 *     device status word (HPA_DEVICE_*), read back with hpa_read_status.
 *   - Shapes: head_dim D in {64, 128}; page (tile) size 64 tokens; GQA group
 *     G = num_q_heads / num_kv_heads in 1 .. 32 (G x query tokens <= 32 rows per
 *     kv head, padded to whole MMA n-tiles of 8; the fused prologue G <= 16).
 *
 * Tensor layouts (row-major, innermost last):
 *   q, q_raw, out        [batch][num_q_heads][D]
 *   k_raw, v_raw         [batch][num_kv_heads][D]
 *   k_cache, v_cache     [num_pages][num_kv_heads][64][D]   one (page, kv head)
 *                        tile is one contiguous 64 x D block
 *   k_scale, v_scale     [num_pages][num_kv_heads] fp32      (FP8 caches only)
 *   page_table           [batch][pt_stride] int32: physical page of tile t of
 *                        sequence b; entries past a sequence's last tile are
 *                        never read
 *   seq_lens             [batch] int32: tokens attended this step (after the
 *                        prologue appended the new one)
 *   positions            [batch] int32: 0-based index of the new token (the
 *                        length before the append)
 *   Token j of sequence b lives in row j % 64 of page page_table[b][j / 64].
 *
 * Sources.  The method is the HPC-Ops attention backend as reported on the
 * web pages this library restates: xiaodao.ai "HPC-Ops TPOT -48.8%"
 * (Attention section: live KV cut into 64-token tiles, the global task list
 * spread as evenly as possible over persistent CTAs, versus static split-KV
 * with a fixed split count or a fixed split size), bitbyai.com "vLLM x
 * HPC-Ops" (Attention Backend: per-step load-balanced scheduler; RoPE,
 * query-key normalisation and KV-write fused into a prologue), openai-hub.com
 * news/688 (the illustrative paged attention call) and aipuzi.cn "HPC-Ops"
 * (section 2.3: native BF16/FP8).
 */
#ifndef HPA_H
#define HPA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HPA_API __attribute__((visibility("default")))
#else
#define HPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HPA_OK = 0,
  HPA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent shapes */
  HPA_ERR_UNSUPPORTED = 2,  /* a shape outside the supported set (see above) */
  HPA_ERR_WORKSPACE = 3,    /* workspace too small or misaligned */
  HPA_ERR_CUDA = 4          /* a CUDA runtime/driver call or launch failed;
                               hpa_last_cuda_error() names it */
} hpa_status;

typedef enum { HPA_KV_BF16 = 0, HPA_KV_FP8_E4M3 = 1 } hpa_kv_dtype;
typedef enum { HPA_OUT_BF16 = 0, HPA_OUT_F32 = 1 } hpa_out_dtype;

/* Plan kinds.  DYNAMIC is the method; the two STATIC kinds are the static
 * split-KV schedules it is measured against, fed to the same run kernel
 * (xiaodao.ai "HPC-Ops TPOT -48.8%", Attention section).  LENGTH_AWARE is
 * DYNAMIC with the cut points moved so that short sequences stay whole and
 * long ones are cut into pieces of at least `param` tiles (bitbyai.com "vLLM
 * x HPC-Ops", Attention Backend: nearly-finished short requests first, long
 * ones spread over the grid); see hpa_decode_plan. */
typedef enum {
  HPA_PLAN_DYNAMIC = 0,        /* param unused; tail and cost weights: hpa_decode_plan_shape */
  HPA_PLAN_STATIC_NSPLIT = 1,  /* param = splits per (seq, kv head); 0 = ceil(num_ctas / (B Hkv)) */
  HPA_PLAN_STATIC_CHUNK = 2,   /* param = tiles per split; 0 = ceil(T_max / ceil(num_ctas / Hkv)) */
  HPA_PLAN_LENGTH_AWARE = 3    /* param = smallest end piece of a cut segment, tiles; 0 = 4 */
} hpa_plan_kind;

/* Shape of the run-time tail of the DYNAMIC and LENGTH_AWARE plans (see
 * hpa_decode_plan), for U units over P persistent CTAs: if tail_den > 0 and
 * U >= tail_min * P, the last Ut = min(floor(U / tail_den), U - P) units are
 * cut into M = min(tail_chunks * P, Ut) chunks; otherwise there is no tail.
 * These are this library's tuning choices, not part of the method: the pages
 * fix only that the global tile list is spread as evenly as possible over the
 * persistent CTAs, which every shape does, and no tail is that even spread
 * with nothing left to run time.  A tail evens out the CTAs' unequal shares
 * of HBM bandwidth, which matters once each CTA streams many tiles; on a
 * batch of a few tiles per CTA its one-tile chunks cost more in partials and
 * merge work than they save, hence tail_min.  hpa_decode_plan, the in-kernel
 * plans (hpa_decode_step*) and hpa_decode_noalloc use the defaults;
 * hpa_decode_plan_shape takes all three as arguments.  HPA_TAIL_CHUNKS_MAX
 * bounds tail_chunks (the workspace has room for that many chunks per CTA). */
#define HPA_TAIL_DEN_DEFAULT 8
#define HPA_TAIL_CHUNKS_DEFAULT 4
#define HPA_TAIL_MIN_DEFAULT 32
#define HPA_TAIL_CHUNKS_MAX 4

/* Cost weights of the primary ranges of the DYNAMIC and LENGTH_AWARE plans
 * (see hpa_decode_plan): every unit costs unit_cost and the last unit of each
 * (sequence, kv head) segment end_cost more -- the segment's end, where its
 * state is handed over and combined, takes time of its own, so a range of
 * many short segments runs longer than one of as many units of a long one.
 * The primary ranges split the primary units' total cost evenly, provided
 * that total is at least (unit_cost + end_cost) times the CTA count, so that
 * no primary range is empty; below that, and always with end_cost = 0, they
 * split the units themselves evenly.  Like the tail, these are this
 * library's tuning, not part of the method.  hpa_decode_plan uses
 * (HPA_COST_UNIT_DEFAULT, HPA_COST_END_DEFAULT) = (1, 0), and so do the
 * in-kernel plans (hpa_decode_step*, hpa_decode_noalloc) for bf16 caches; for
 * e4m3 caches, whose 64-token tiles stream in half the time of a bf16 tile so
 * that a segment end weighs twice as much, they use (1,
 * HPA_COST_END_DEFAULT_FP8) = (1, 2) (measured: a batch of many short
 * sequences runs 16 % faster, long ones as before).  hpa_decode_plan_shape
 * takes any weights, each in 0 .. HPA_COST_MAX (unit_cost >= 1); with (1, 2)
 * it gives an e4m3 run the in-kernel plan's ranges. */
#define HPA_COST_UNIT_DEFAULT 1
#define HPA_COST_END_DEFAULT 0
#define HPA_COST_END_DEFAULT_FP8 2
#define HPA_COST_MAX 4

/* Bits of the device status word (hpa_read_status). */
#define HPA_DEVICE_LEN_CLAMPED 0x1  /* a seq_len < 0 or > pt_stride * 64 was clamped */
#define HPA_DEVICE_BAD_PAGE 0x2     /* a page id outside [0, num_pages) was skipped  */
#define HPA_DEVICE_BAD_PLAN 0x4     /* run found no plan, or one for other shapes    */
#define HPA_DEVICE_BAD_POSITION 0x8 /* prologue: position outside the page table     */
#define HPA_DEVICE_TIMEOUT 0x10     /* a pipeline wait gave up after 2 s (results void) */

/* Human-readable name of a status code (static string, never NULL). */
HPA_API const char* hpa_status_string(hpa_status status);

/* Text of the last CUDA error seen by a call on this host thread ("" if none). */
HPA_API const char* hpa_last_cuda_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
HPA_API int hpa_version(void);

/* Number of persistent CTAs for `device`: two per SM (296 on B200), which
 * the run kernel executes as two co-resident CTAs per SM.  The environment
 * variable HPA_NUM_CTAS (a decimal count 1 .. 65536) overrides it; other
 * values of it are ignored.  Returns -1 if the device cannot be queried. */
HPA_API int hpa_default_num_ctas(int device);

/* Persistent CTA count (num_ctas of hpa_decode_plan) that matches how many
 * run-kernel CTAs fit at once for this head geometry; a dynamic plan for more
 * CTAs than fit would leave part of its primary ranges to a second wave.
 * Up to 32 query rows per kv head (G * q_tokens) two fit per SM, and this is
 * hpa_default_num_ctas.  Returns -1 on invalid arguments (more than 32 rows)
 * or if the device cannot be queried. */
HPA_API int hpa_decode_num_ctas(int device, int num_q_heads, int num_kv_heads, int q_tokens);

/* Grid (CTA count) of the run kernel under a plan: num_ctas for DYNAMIC and
 * LENGTH_AWARE, B * Hkv * S for STATIC_NSPLIT, B * Hkv * ceil(T_max / C) for STATIC_CHUNK
 * (T_max = ceil(max_seq_len / 64), S and C the resolved params).  Host only;
 * returns -1 on invalid arguments. */
HPA_API int hpa_plan_grid(hpa_plan_kind kind, int batch, int num_kv_heads, int num_ctas, int param,
                  int max_seq_len);

/* Bytes of device workspace that a plan of this kind over `grid` CTAs and
 * the matching run need.  Host only; returns 0 on invalid arguments. */
HPA_API size_t hpa_decode_workspace_size(hpa_plan_kind kind, int batch, int num_kv_heads,
                                         int num_q_heads, int head_dim, int grid);

/* Byte offsets of the workspace regions, for inspection by tests and tools:
 * offsets[0..6] = header (int32[32]: magic, status, units, grid, kind, batch,
 * kv heads, group, head_dim, tiles, ranges V, next tail chunk, finished CTAs,
 * tail_den, tail_chunks, tail_min (0 for the static kinds), split segments
 * listed for the merge (two counts, by step parity), the step parity,
 * unit_cost, end_cost (0 for the static kinds), then zeros), lens,
 * tile_start, range descriptors (int32 x8 per range: u_begin, u_end, then
 * the sequence, kv head, tile and tile count of its first unit, 0, 0),
 * segment descriptors (int32 x2 per (sequence, kv head): slot of its first
 * partial or -1, number of ranges holding it), partial (m, l), partial acc;
 * offsets[7] = total size.  Range v keeps the partial of its first segment
 * in slot 2v and that of its last segment in slot 2v + 1.
 * Returns HPA_OK or HPA_ERR_INVALID_ARG. */
HPA_API hpa_status hpa_workspace_layout(hpa_plan_kind kind, int batch, int num_kv_heads,
                                        int num_q_heads, int head_dim, int grid,
                                        size_t offsets[8]);

/*
 * hpa_decode_plan -- per-step tile plan (xiaodao.ai "HPC-Ops TPOT -48.8%",
 * Attention section; bitbyai.com "vLLM x HPC-Ops", Attention Backend).
 *
 * Cuts every sequence's live KV into 64-token tiles.  A unit is one
 * (sequence b, kv head g, tile t); the global list orders units by b, g, t,
 * and the plan cuts it into contiguous ranges.  DYNAMIC (P = num_ctas
 * persistent CTAs, U units): if U <= P, CTA c < U takes unit c; otherwise the
 * last Ut units (Ut from the tail shape above: min(floor(U/8), U - P) by
 * default when U >= 32 P, else 0) form M tail chunks (min(4P, Ut) by default)
 * [U1 + floor(jUt/M), U1 + floor((j+1)Ut/M)) and the first U1 = U - Ut units
 * the P primary ranges.  With the cost weights q = unit_cost, e = end_cost
 * (above) and K(x) = q x + e n(x), n(x) the number of segments whose last
 * unit comes before unit x, primary range c is [x_c, x_(c+1)) where x_c is
 * the largest x <= U1 with P K(x) <= c K(U1), if K(U1) >= (q + e) P; else,
 * and for e = 0, it is [floor(cU1/P), floor((c+1)U1/P)).  CTA c runs primary
 * range c, then takes tail chunks in order from a counter as it finishes, so
 * CTAs that got more HBM bandwidth do more of the tail.  A short sequence
 * lands whole in one range; a long one is spread over many.  The STATIC
 * kinds give one CTA per (segment, split) instead.
 *
 * LENGTH_AWARE (m = param, or 4 if 0): the DYNAMIC ranges with every cut point
 * x moved as follows.  If x falls strictly inside a segment [s0, s1) (the
 * units of one (sequence, kv head)) and would leave a piece of fewer than m
 * tiles (x - s0 < m or s1 - x < m), it moves to the nearer end of the segment
 * (s0 on a tie).  A segment of fewer than 2m tiles is never cut: it runs
 * whole in one range and finishes without partials or a merge.  A longer one
 * is spread as under DYNAMIC, but its first and last pieces have at least m
 * tiles.  Ranges stay contiguous and in order; some may become empty.
 * m = 1 gives DYNAMIC's ranges exactly.  Same workspace size and run-time
 * tail as DYNAMIC; hpa_decode_run with kind = LENGTH_AWARE.
 *
 *   seq_lens     device [batch] int32; values are clamped to [0, pt_stride*64]
 *                (HPA_DEVICE_LEN_CLAMPED).  A sequence of length 0 gets a zero
 *                output row from hpa_decode_run.
 *   num_ctas     persistent CTA count (hpa_default_num_ctas), >= 1.
 *   max_seq_len  host upper bound on every seq_len; sizes the STATIC_CHUNK
 *                grid (ignored otherwise, may be 0).
 *   workspace    device, >= hpa_decode_workspace_size(kind, ..., grid)
 *                bytes, 256-byte aligned.  The plan rewrites everything the
 *                run reads.
 *   grid_out     host; receives the grid hpa_decode_run must be given.
 *
 * Recompute the plan whenever seq_lens change (every decode step).  A run
 * must use the workspace of the plan made for its step; two steps in flight
 * at once need two workspaces.
 */
HPA_API hpa_status hpa_decode_plan(const int32_t* seq_lens, int batch, int num_kv_heads,
                           int num_q_heads, int head_dim, int pt_stride, hpa_plan_kind kind,
                           int num_ctas, int param, int max_seq_len, void* workspace,
                           size_t ws_bytes, int* grid_out, void* stream);

/*
 * hpa_decode_plan_shape -- hpa_decode_plan for the DYNAMIC or LENGTH_AWARE
 * kind with the run-time tail's shape and the cost weights of the primary
 * ranges given explicitly (xiaodao.ai "HPC-Ops TPOT -48.8%", Attention
 * section: the even spread of the tile list; bitbyai.com "vLLM x HPC-Ops",
 * Attention Backend: progress evaluated at run time).
 *
 *   tail_den     0 .. 2^20: the tail holds min(floor(U / tail_den), U - P)
 *                units; 0 = no tail (the primary ranges are the even
 *                partition of all U units).
 *   tail_chunks  1 .. HPA_TAIL_CHUNKS_MAX: the tail is cut into
 *                min(tail_chunks * P, Ut) chunks (ignored if the tail is empty).
 *   tail_min     0 .. 2^20: no tail unless U >= tail_min * P.
 *   unit_cost    1 .. HPA_COST_MAX: cost of one unit.
 *   end_cost     0 .. HPA_COST_MAX: extra cost of a segment's last unit;
 *                0 = the primary ranges split the units evenly.
 *   the rest     as for hpa_decode_plan (max_seq_len is not needed).
 * Any other kind, or a parameter out of range, returns HPA_ERR_INVALID_ARG.
 * The workspace size and hpa_decode_run's arguments do not depend on the
 * shape.  hpa_decode_plan(kind, ...) equals hpa_decode_plan_shape(kind, ...,
 * HPA_TAIL_DEN_DEFAULT, HPA_TAIL_CHUNKS_DEFAULT, HPA_TAIL_MIN_DEFAULT,
 * HPA_COST_UNIT_DEFAULT, HPA_COST_END_DEFAULT, ...).
 */
HPA_API hpa_status hpa_decode_plan_shape(const int32_t* seq_lens, int batch, int num_kv_heads,
                                         int num_q_heads, int head_dim, int pt_stride,
                                         hpa_plan_kind kind, int num_ctas, int param,
                                         int tail_den, int tail_chunks, int tail_min,
                                         int unit_cost, int end_cost, void* workspace,
                                         size_t ws_bytes, int* grid_out, void* stream);

/*
 * hpa_decode_run -- persistent paged GQA decode attention with split-KV
 * log-sum-exp merge (xiaodao.ai "HPC-Ops TPOT -48.8%", Attention section:
 * persistent CTAs consume 64-token tiles; a sequence split over CTAs is
 * merged from per-split partials).
 *
 * For sequence b and query head h (kv head g = h / G):
 *     out[b][h] = sum_j softmax_j(softmax_scale * <q[b][h], K_b[j, g]>) V_b[j, g]
 * over j < seq_lens[b] as captured by the plan.  Computed in fp32 with
 * bf16 (or f16 for FP8 caches) tensor-core products.
 *
 *   q            device bf16 [batch][num_q_heads][D]
 *   k_cache, v_cache  device [num_pages][num_kv_heads][64][D]; bf16, or e4m3
 *                codes when kv_dtype = HPA_KV_FP8_E4M3.  16-byte aligned.
 *   k_scale, v_scale  device fp32 [num_pages][num_kv_heads] dequantisation
 *                scales (value = code * scale); NULL for bf16 caches.
 *   page_table   device int32 [batch][pt_stride]; ids outside
 *                [0, num_pages) are skipped (HPA_DEVICE_BAD_PAGE).
 *   out          device [batch][num_q_heads][D], bf16 or fp32 (out_dtype).
 *   kind, grid   the kind and grid_out of the plan that filled `workspace`.
 *   workspace    the plan's workspace; its partial regions are rewritten by
 *                the run.
 * Splits of one (sequence, kv head) leave fp32 partials in the workspace; a
 * second kernel launched by this call merges them in split order, so results
 * do not depend on CTA timing.
 */
HPA_API hpa_status hpa_decode_run(const void* q, const void* k_cache, const void* v_cache,
                          const float* k_scale, const float* v_scale, hpa_kv_dtype kv_dtype,
                          const int32_t* page_table, int pt_stride, int num_pages, void* out,
                          hpa_out_dtype out_dtype, int batch, int num_q_heads,
                          int num_kv_heads, int head_dim, float softmax_scale,
                          hpa_plan_kind kind, int grid, void* workspace, size_t ws_bytes,
                          void* stream);

/*
 * hpa_decode_run_multi -- hpa_decode_run for T = q_tokens new query tokens per
 * sequence (a draft token to verify, or multi-token-prediction heads), causal
 * among themselves.  The pages' attention API takes variable-length queries
 * per sequence (openai-hub.com news/688: attention(q, k, v, cu_seqlens, ...,
 * kv_cache_layout="paged")); this is its fixed-T decode form.
 *
 * The T tokens are the last T of each sequence and are already in the cache
 * (seq_lens counts them).  Query token i (0 <= i < T) of sequence b sits at
 * position seq_lens[b] - T + i and attends to positions 0 .. seq_lens[b] -
 * T + i:
 *     out[b][i][h] = sum_{j <= L_b - T + i} softmax_j(scale <q[b][i][h], K_b[j, g]>) V_b[j, g]
 * A query that sees no token (seq_lens[b] < T - i) gets a zero row.
 *
 *   q, out       device [batch][q_tokens][num_q_heads][D] (bf16 q; bf16 or
 *                fp32 out).
 *   q_tokens     1 .. 16 with (num_q_heads / num_kv_heads) * q_tokens <= 32:
 *                the G * T query rows of a kv head share one pass over its
 *                tiles (HPA_ERR_UNSUPPORTED otherwise).  Above 16 rows the
 *                kernel keeps one deposit buffer and two stages per CTA so
 *                that two CTAs still fit an SM (hpa_decode_num_ctas).
 *   kind, grid, workspace  from hpa_decode_plan called with num_q_heads *
 *                q_tokens in place of num_q_heads (the plan and the workspace
 *                count G * T rows per kv head); size the workspace the same way.
 *   the rest     as for hpa_decode_run; q_tokens = 1 is hpa_decode_run.
 */
HPA_API hpa_status hpa_decode_run_multi(const void* q, const void* k_cache, const void* v_cache,
                                        const float* k_scale, const float* v_scale,
                                        hpa_kv_dtype kv_dtype, const int32_t* page_table,
                                        int pt_stride, int num_pages, void* out,
                                        hpa_out_dtype out_dtype, int batch, int q_tokens,
                                        int num_q_heads, int num_kv_heads, int head_dim,
                                        float softmax_scale, hpa_plan_kind kind, int grid,
                                        void* workspace, size_t ws_bytes, void* stream);

/*
 * hpa_decode_step -- one decode step with the dynamic plan made inside the
 * decode kernel: hpa_decode_plan(kind = DYNAMIC, num_ctas) followed by
 * hpa_decode_run_multi, in two launches instead of three (xiaodao.ai
 * "HPC-Ops TPOT -48.8%", Attention section: the per-step load-balanced tile
 * plan; here each persistent CTA scans the lengths itself and derives its own
 * ranges from the same closed forms, so the step needs no plan kernel and no
 * wait for one).  Same partition, same partial slots and merge order, hence
 * the same bits as the two-call path -- for an e4m3 cache that path's plan
 * is hpa_decode_plan_shape with the cost weights (HPA_COST_UNIT_DEFAULT,
 * HPA_COST_END_DEFAULT_FP8) (see the cost weights above).
 *
 *   seq_lens     device [batch] int32, as for hpa_decode_plan.
 *   batch        1 .. 512 (the tile offsets live in shared memory;
 *                HPA_ERR_UNSUPPORTED beyond: use hpa_decode_plan + run).
 *   num_ctas     persistent CTAs (hpa_decode_num_ctas), 1 .. 65536; also the
 *                grid the workspace is sized for.
 *   workspace    >= hpa_decode_workspace_size(HPA_PLAN_DYNAMIC, batch,
 *                num_kv_heads, num_q_heads * q_tokens, head_dim, num_ctas)
 *                bytes, 256-byte aligned, zero-filled before its first use
 *                (or last written by hpa_decode_plan); every dynamic run
 *                leaves its run-time counters at zero for the next step, and
 *                the merge empties the list of split segments the decode
 *                kernel makes for it.  (After a call that returned
 *                HPA_ERR_CUDA, zero the workspace or plan on it again.)  The
 *                plan fields of the header and the segment descriptors are
 *                written as hpa_decode_plan writes them; the range
 *                descriptors are not.  Status bits accumulate until a
 *                hpa_decode_plan on the workspace clears them.
 *   the rest     as for hpa_decode_run_multi (q_tokens = 1: single-token).
 */
HPA_API hpa_status hpa_decode_step(const int32_t* seq_lens, const void* q, const void* k_cache,
                                   const void* v_cache, const float* k_scale,
                                   const float* v_scale, hpa_kv_dtype kv_dtype,
                                   const int32_t* page_table, int pt_stride, int num_pages,
                                   void* out, hpa_out_dtype out_dtype, int batch, int q_tokens,
                                   int num_q_heads, int num_kv_heads, int head_dim,
                                   float softmax_scale, int num_ctas, void* workspace,
                                   size_t ws_bytes, void* stream);

/*
 * hpa_decode_run_prologue -- hpa_decode_run with the decode prologue fused
 * into the persistent kernel (bitbyai.com "vLLM x HPC-Ops", Attention
 * Backend: RoPE, query-key normalisation and the KV write fused into one
 * prologue to save launches and HBM round trips; here the prologue does not
 * even get its own launch).
 *
 * Equivalent to hpa_kv_prologue(q_raw, k_raw, v_raw, q_gamma, k_gamma, eps,
 * rope_theta, positions = seq_lens - 1, ...) followed by hpa_decode_run on
 * its q_out, with the same bits in the output, in the written K/V slots and
 * in q_out: every CTA that starts a piece of (sequence, kv head) normalises
 * and rotates that head group's raw query rows in shared memory, and the CTA
 * whose range holds a sequence's last tile computes the new token's K and V
 * rows, stores them in their cache slot (position seq_len - 1) and only then
 * loads that tile.
 *
 *   q_raw, k_raw, v_raw  device bf16 [batch][Hq][D] / [batch][Hkv][D], the
 *                new token's pre-norm rows; 16-byte aligned.
 *   q_gamma, k_gamma, eps, rope_theta  as for hpa_kv_prologue.
 *   k_cache, v_cache  device bf16 caches (written at the new token's slot).
 *   q_out        optional (NULL: not written) device bf16 [batch][Hq][D]:
 *                the normalised, rotated queries.  Rows of sequences of
 *                length 0 are not written.
 *   the rest     as for hpa_decode_run; the plan's seq_lens are the
 *                post-append lengths (the new token included).
 * bf16 caches only (the call has no kv_dtype argument).  A length the plan
 * clamped (HPA_DEVICE_LEN_CLAMPED) voids that step's output and K/V writes.
 */
HPA_API hpa_status hpa_decode_run_prologue(
    const void* q_raw, const void* k_raw, const void* v_raw, const float* q_gamma,
    const float* k_gamma, float eps, float rope_theta, void* k_cache, void* v_cache, void* q_out,
    const int32_t* page_table, int pt_stride, int num_pages, void* out, hpa_out_dtype out_dtype,
    int batch, int num_q_heads, int num_kv_heads, int head_dim, float softmax_scale,
    hpa_plan_kind kind, int grid, void* workspace, size_t ws_bytes, void* stream);

/*
 * hpa_decode_step_prologue -- hpa_decode_step with the prologue of
 * hpa_decode_run_prologue: a whole decode step -- RMSNorm + RoPE of q and of
 * the new K row, the new token's K/V cache write, the dynamic tile plan,
 * attention and the split merge -- in two launches (bitbyai.com "vLLM x
 * HPC-Ops", Attention Backend: the fused prologue; xiaodao.ai "HPC-Ops TPOT
 * -48.8%", Attention section: the per-step plan).  Same bits as
 * hpa_kv_prologue + hpa_decode_plan + hpa_decode_run.
 *
 * Arguments as for hpa_decode_run_prologue, with seq_lens (post-append
 * lengths), num_ctas and the workspace rules of hpa_decode_step (batch <= 512,
 * workspace zero-filled before its first use).
 */
HPA_API hpa_status hpa_decode_step_prologue(
    const int32_t* seq_lens, const void* q_raw, const void* k_raw, const void* v_raw,
    const float* q_gamma, const float* k_gamma, float eps, float rope_theta, void* k_cache,
    void* v_cache, void* q_out, const int32_t* page_table, int pt_stride, int num_pages,
    void* out, hpa_out_dtype out_dtype, int batch, int num_q_heads, int num_kv_heads,
    int head_dim, float softmax_scale, int num_ctas, void* workspace, size_t ws_bytes,
    void* stream);

/*
 * hpa_decode_step_lse -- hpa_decode_step that also returns each output row's
 * log-sum-exp, so that steps run over different parts of the same sequences
 * (the GPUs of a tensor-parallel group holding different page ranges of every
 * sequence, openai-hub.com news/688; a shared prefix and a private suffix)
 * can be combined with hpa_merge_states.  This is the split-KV recombination
 * of xiaodao.ai "HPC-Ops TPOT -48.8%" (Attention section) carried across
 * calls.
 *
 *   lse          device fp32 [batch][q_tokens][num_q_heads], 4-byte aligned,
 *                required: lse[b][i][h] = log sum_j exp(softmax_scale *
 *                q[b][i][h] . k_j) over the keys row (b, i, h) attends, in
 *                natural-log units; -inf (and a zero output row) where the row
 *                attends no key (a sequence of length 0).
 *   the rest     as for hpa_decode_step; `out` holds the normalised rows.
 * Use HPA_OUT_F32 for `out` when the rows are merged afterwards.
 */
HPA_API hpa_status hpa_decode_step_lse(const int32_t* seq_lens, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const float* k_scale, const float* v_scale,
                                       hpa_kv_dtype kv_dtype, const int32_t* page_table,
                                       int pt_stride, int num_pages, void* out,
                                       hpa_out_dtype out_dtype, float* lse, int batch,
                                       int q_tokens, int num_q_heads, int num_kv_heads,
                                       int head_dim, float softmax_scale, int num_ctas,
                                       void* workspace, size_t ws_bytes, void* stream);

/*
 * hpa_merge_states -- log-sum-exp merge of attention states computed over
 * disjoint key sets of the same rows (the recombination step of split-KV
 * decode, xiaodao.ai "HPC-Ops TPOT -48.8%", Attention section, across calls
 * or GPUs).  For every row r, with M = max_i lse_i[r] and w_i = exp(lse_i[r]
 * - M):
 *
 *     out[r]     = sum_i (w_i / sum_k w_k) o_i[r]     (folded in index order)
 *     lse_out[r] = M + log sum_i w_i
 *
 * A state with lse = -inf contributes nothing (its o row is loaded but not
 * used, so it may hold anything, NaN included); a row whose states are all
 * -inf gets out = 0 and lse_out = -inf.
 *
 *   o_parts      HOST array of num_states device pointers, each fp32
 *                [rows][head_dim], 16-byte aligned (hpa_decode_step_lse with
 *                HPA_OUT_F32).  A pointer may address a peer GPU's memory
 *                mapped into the current context: the kernel reads it with
 *                plain global loads.  Every buffer (states, out, lse_out) must
 *                be reachable from the current device -- its own memory,
 *                managed memory, mapped pinned host memory, or a peer's
 *                memory with peer access enabled; a pageable host pointer or
 *                an unknown address returns HPA_ERR_INVALID_ARG (a failed
 *                driver query, HPA_ERR_CUDA) before anything is enqueued.  The
 *                check is a driver query per new pointer, remembered per host
 *                thread; it cannot tell whether peer access was enabled.
 *   lse_parts    HOST array of num_states device pointers, each fp32 [rows].
 *   num_states   1 .. 16 (HPA_ERR_UNSUPPORTED beyond).
 *   rows         >= 0; 0 enqueues nothing.
 *   head_dim     64 or 128.
 *   out          device [rows][head_dim], bf16 (8-byte aligned) or fp32
 *                (16-byte aligned) per out_dtype; may not alias an o part.
 *   lse_out      optional (NULL: not written) device fp32 [rows].
 * Launched with programmatic dependent launch on `stream`, so it can start
 * while the kernel before it drains.
 */
HPA_API hpa_status hpa_merge_states(const float* const* o_parts, const float* const* lse_parts,
                                    int num_states, long long rows, int head_dim, void* out,
                                    hpa_out_dtype out_dtype, float* lse_out, void* stream);

/*
 * hpa_kv_prologue -- fused RMSNorm + RoPE + KV write for the new token of
 * each sequence (bitbyai.com "vLLM x HPC-Ops", Attention Backend: RoPE,
 * query-key normalisation and KV-write fused into one prologue).
 *
 * For sequence b at position p = positions[b]:
 *   q_out[b][h]  = RoPE(RMSNorm(q_raw[b][h]; q_gamma), p)       for every h
 *   K slot (b,g) = RoPE(RMSNorm(k_raw[b][g]; k_gamma), p)       rounded to bf16
 *   V slot (b,g) = v_raw[b][g]                                  bit copy
 * with RMSNorm(x; w)_i = x_i / sqrt(mean(x^2) + eps) * w_i over one head's D
 * elements and rotate-half RoPE over the full head: for i < D/2,
 * phi = p * theta^(-2i/D), (x_i, x_{i+D/2}) -> (x_i cos phi - x_{i+D/2} sin phi,
 * x_{i+D/2} cos phi + x_i sin phi).  The slot is row p % 64 of page
 * page_table[b][p / 64], kv head g.  The step then attends p + 1 tokens.
 *
 *   q_raw, k_raw, v_raw  device bf16, layouts above.
 *   q_gamma, k_gamma     device fp32 [D], shared by all heads.
 *   positions            device int32 [batch]; a position whose page-table
 *                        entry is missing or out of range skips the K/V write
 *                        and sets HPA_DEVICE_BAD_POSITION in *status.
 *   k_cache, v_cache     device bf16 caches, written in place (one row per
 *                        (b, g); nothing else is touched).
 *   q_out                device bf16 [batch][num_q_heads][D].
 *   status               device int32 word ORed with HPA_DEVICE_* bits, or NULL.
 */
HPA_API hpa_status hpa_kv_prologue(const void* q_raw, const void* k_raw, const void* v_raw,
                           const float* q_gamma, const float* k_gamma, float eps,
                           float rope_theta, const int32_t* positions,
                           const int32_t* page_table, int pt_stride, void* k_cache,
                           void* v_cache, void* q_out, int batch, int num_q_heads,
                           int num_kv_heads, int head_dim, int num_pages, int32_t* status,
                           void* stream);

/*
 * hpa_decode_noalloc -- one decode step (plan + run, dynamic plan) for callers
 * that must not allocate device memory while they run it: code inside a
 * device memory pool that may not grow after start-up, code whose allocator
 * belongs to another framework and is out of reach where the step is issued,
 * or a plain C program that keeps cudaMalloc off its hot path.  The pages
 * have no counterpart of this call; it exists for such integrations.
 *
 * Arguments are those of hpa_decode_plan + hpa_decode_run with the dynamic
 * plan; num_ctas = 0 means one CTA per SM (the device's SM count: unlike
 * hpa_default_num_ctas, the HPA_NUM_CTAS variable does not change it, since
 * the CTA count sizes the scratch).  Instead of a caller workspace the
 * step uses a library-owned static device array of HPA_NOALLOC_SCRATCH_BYTES
 * (16 MiB), which every GPU that loads the library holds until the process
 * exits.  A step whose workspace would exceed it (see
 * hpa_decode_workspace_size) returns HPA_ERR_WORKSPACE before any CUDA call.
 * The call allocates nothing: no cudaMalloc, cudaFree or allocating library
 * routine.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and the SM count with that device current; make that
 * first call before any stream capture.  All calls share the array and it
 * keeps the last call's contents; every call rewrites everything it reads
 * (up to 512 sequences the plan is made inside the decode kernel, as
 * hpa_decode_step does; beyond, hpa_decode_plan runs first) and leaves the
 * run-time counters at zero, so stale contents never reach a result, but
 * calls that overlap on the GPU (unordered streams) race on the array.  The
 * array's address is cached per device for the life of the process: calls
 * must not cross a cudaDeviceReset (or any other end of the device's primary
 * context).  Device-side problems (a page id out of range, a clamped length,
 * a timed-out wait) set bits in the array's status word, read with
 * hpa_noalloc_read_status.
 */
#define HPA_NOALLOC_SCRATCH_BYTES (16u << 20)
HPA_API hpa_status hpa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                      const float* k_scale, const float* v_scale,
                                      hpa_kv_dtype kv_dtype, const int32_t* page_table,
                                      int pt_stride, int num_pages, const int32_t* seq_lens,
                                      void* out, hpa_out_dtype out_dtype, int batch,
                                      int num_q_heads, int num_kv_heads, int head_dim,
                                      float softmax_scale, int num_ctas, void* stream);

/* The status word (HPA_DEVICE_* bits) of hpa_decode_noalloc's static array on
 * the current device, copied to *status_out (host) after the work queued on
 * `stream` so far; with clear != 0 the word is then reset to 0 (in stream
 * order).  The bits of every call accumulate until cleared, except that a
 * call of more than 512 sequences starts by rewriting the word with its own
 * plan's bits.  Synchronises the stream; allocates nothing.  The first call
 * on a device does the array set-up described at hpa_decode_noalloc. */
HPA_API hpa_status hpa_noalloc_read_status(int32_t* status_out, int clear, void* stream);

/* Copies the device status word of a plan's workspace to *status_out (host)
 * after the work queued on `stream` so far; synchronises the stream. */
HPA_API hpa_status hpa_read_status(const void* workspace, int32_t* status_out, void* stream);

/*
 * hpa_read_cta_times -- per-CTA timeline of the last run on a workspace, for
 * measuring how evenly the plan loaded the persistent CTAs (the tail idle time
 * the dynamic scheduler exists to remove: bitbyai.com "vLLM x HPC-Ops",
 * Attention Backend, static splits leave GPU compute units idle).
 *
 * Every run-kernel launch (hpa_decode_run*, hpa_decode_step*) writes, for each
 * of its `grid` CTAs c, four uint64 values to the workspace:
 *   times_out[4c + 0]  %globaltimer (ns) when CTA c started its work (after
 *                      waiting for the kernel before it)
 *   times_out[4c + 1]  when its producer warp had issued its last tile
 *   times_out[4c + 2]  when its epilogue warp had written its last result
 *   times_out[4c + 3]  units (tiles of one kv head) it streamed
 * The shape arguments are those the workspace was sized with
 * (hpa_decode_workspace_size); times_out is a HOST array of 4 * grid values.
 * Synchronises the stream.  Values of CTAs of an aborted run are undefined.
 */
HPA_API hpa_status hpa_read_cta_times(const void* workspace, hpa_plan_kind kind, int batch,
                                      int num_kv_heads, int num_q_heads, int head_dim, int grid,
                                      uint64_t* times_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HPA_H */
