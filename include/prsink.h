/*
 * prsink.h - C ABI of the B200 (sm_100a) library for LiveAnimate's PR-Sink per-block step.
 *
 * Sources (web pages about arXiv 2608.11745 "LiveAnimate: Stable Long-Form Streaming Human
 * Animation in Real-Time"), cited below by tag:
 *   [digest]    paper.rainbus.top/paper/2608.11745 digest; paragraphs "pipeline" (with its
 *               inference clause), "novelty" (points 2-4), "weaknesses", "reproducibility".
 *   [explainer] papers.ananclaw.com explainer, section "Pose-Retrieval Sink Attention (PR-Sink)".
 *   [abstract]  HF papers abstract (Chinese translation, bittide mirror).
 *   [news]      jiazhuangai.com article, section "three key breakthroughs", item 1.
 *
 * Conventions shared by every call:
 *   - All pointers except `const prsink_layout*` point to DEVICE memory owned by the caller;
 *     the library keeps no allocation of its own.  bf16 buffers are passed as void*.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is asynchronous
 *     on that stream; decisions (retrieved slot, bank action) stay on the device, so a
 *     sequence of calls needs no host synchronisation.
 *   - Return value: PRSINK_OK (0) or a negative PRSINK_ERR_* code.  Invalid arguments are
 *     rejected on the host before anything is launched.  No C++ exception crosses the ABI.
 *   - Device-side waits are bounded.  A wait that runs out records PRSINK_ERR_TIMEOUT in a
 *     device status word; prsink_sync_status() reads and clears it.  There is ONE status word
 *     per device, shared by every stream and host thread that uses the library on it: a
 *     timeout raised by a kernel on stream A is reported (and cleared) by a
 *     prsink_sync_status() call made for stream B.
 *
 * Cache layout (the "slot-indexed" cache).  For one layer, K and V caches are each
 * bf16 [H][T][d] (head-major, d contiguous).  Physical key rows are grouped in slots:
 *   slot 0  PRSINK_SLOT_REF      L_ref = ref_frames * L_f rows      (reference image)
 *   slot 1  PRSINK_SLOT_STATIC   L_blk rows                         (first generated block)
 *   slot 2  PRSINK_SLOT_DYNAMIC  L_blk rows                         (pose-retrieved block)
 *   slot 3+s ring slot s         L_blk rows each, s = 0..R-1        (rolling window)
 * with L_f = grid_h*grid_w, L_blk = frames_per_block*L_f and T = L_ref + (2+R)*L_blk.
 * ([explainer] slot diagram [Static][Dynamic][Rolling t-2,t-1,t]; [digest] pipeline formula
 * puts K_ref first; [abstract] static sink = first generated block, dynamic sink = one
 * pose-retrieved block, three-slot rolling window.)  Block b is written into ring slot b mod R.
 *
 * Multi-layer buffers:  cache_kv = bf16 [n_layers][2][H][T][d]   (K then V per layer)
 *                       bank_kv  = bf16 [n_layers][M][2][H][L_blk][d]
 */
#ifndef PRSINK_H
#define PRSINK_H

#ifdef __cplusplus
extern "C" {
#endif

#define PRSINK_OK               0
#define PRSINK_ERR_ARG         (-1)  /* null pointer, bad size, slot out of range          */
#define PRSINK_ERR_ALIGN       (-2)  /* a pointer is not 16-byte aligned                   */
#define PRSINK_ERR_LAUNCH      (-3)  /* CUDA error; text from prsink_last_error()          */
#define PRSINK_ERR_TIMEOUT     (-4)  /* a bounded device wait ran out (see sync_status)    */
#define PRSINK_ERR_UNSUPPORTED (-5)  /* valid but not supported here (e.g. head_dim 96)    */

#define PRSINK_SLOT_REF     0
#define PRSINK_SLOT_STATIC  1
#define PRSINK_SLOT_DYNAMIC 2
#define PRSINK_SLOT_RING0   3
#define PRSINK_MAX_RING     8        /* ring_slots in 1..PRSINK_MAX_RING                    */

#define PRSINK_FP_FRAMES    3        /* [digest] pipeline: three frames per fingerprint     */
#define PRSINK_FP_KEYPOINTS 62       /* [digest] pipeline: 62 keypoints per frame           */
#define PRSINK_FP_CHANNELS  3        /* x, y, confidence ([digest] novelty, point 2)        */
#define PRSINK_FP_DIM       558      /* 3 * 62 * 3                                          */
#define PRSINK_MAX_BANK     32       /* bank size M in 1..PRSINK_MAX_BANK (pages: M = 5)    */

/* Geometry of the bounded cache and of the rotary embedding for one attention layer. */
typedef struct prsink_layout {
  int n_heads;           /* H (40 for the 14B DiT; 1 in the tiny check)                     */
  int head_dim;          /* d, 64 or 128                                                    */
  int grid_h, grid_w;    /* latent tokens per frame = grid_h*grid_w (30x30 at 480x480)     */
  int frames_per_block;  /* B_f latent frames per block (3, [digest] reproducibility)       */
  int ref_frames;        /* latent frames held by the ref sink (1)                         */
  int ring_slots;        /* R, rolling-window slots (3, [explainer])                       */
  int rope_mode;         /* 3 = 3-D RoPE over (t,h,w); 1 = 1-D over the logical token index */
  int rope_split[3];     /* dims given to t, h, w in 3-D mode (44,42,42 for d=128); even     */
  float rope_base;       /* RoPE base (10000)                                               */
  long long block_index; /* b, the block being generated; fixes the ring's age order         */
  unsigned valid_mask;   /* bit i set = slot i holds data (bit 0 ref, 1 static, 2 dynamic,
                            3+s ring slot s); keys of other slots are ignored               */
} prsink_layout;

/* Token counts of a layout: L_f, L_blk, L_ref and T (any out pointer may be NULL).
 * Returns PRSINK_ERR_ARG for an invalid layout. */
int prsink_layout_tokens(const prsink_layout* layout, long long* L_f, long long* L_blk,
                         long long* L_ref, long long* T);

/* PR-Sink attention of the current block for one layer.
 *
 * [digest] pipeline formula: Attn(Q_b,K,V) = softmax(Q_b [K_ref; K_<b]^T / sqrt(d)) [V_ref; V_<b]
 * over the keys the bounded cache holds; [digest] pipeline, inference clause ("RoPE follow"):
 * keys are cached raw (pre-RoPE) and rotated at their current cache position when attended;
 * [digest] novelty, point 4: a reused bank entry is thereby decoupled from its timestamp.
 *
 * Logical key order is [ref; static; dynamic; ring oldest..newest]; frames are numbered
 * 0,1,.. in that order, so ring slot s (holding block b' = s mod R, b' in [b-R+1, b]) sits at
 * frames ref_frames + (2 + b' - (b-R+1)) * B_f ...  A key's 3-D position is (frame, row, col)
 * of its token; its 1-D position is frame*L_f + row*grid_w + col.  Queries sit on the newest
 * ring slot (the current block).  RoPE: interleaved pairs (x[2j], x[2j+1]) of each axis are
 * rotated by pos * base^(-2j/d_axis) (RoFormer); q and k are rotated, v is not.  Scale 1/sqrt(d).
 *
 *   q        bf16 [L_blk][H][d]   raw queries of the current block (token-major)
 *   k_cache  bf16 [H][T][d]       raw keys, slot-indexed (see top of file)
 *   v_cache  bf16 [H][T][d]       values, slot-indexed
 *   out      bf16 [L_blk][H][d]   attention output (written)
 *   lse      f32  [H][L_blk]      natural-log log-sum-exp of the scaled scores, or NULL
 *   dyn_src  int64 scalar or NULL: if given and < 0 the dynamic slot is treated as empty
 *            whatever valid_mask says (lets the retrieval decision stay on the device)
 * Rows of a query with no valid key get out = 0 and lse = -inf.
 * Errors: PRSINK_ERR_ARG (null, sizes), PRSINK_ERR_ALIGN (16 B), PRSINK_ERR_UNSUPPORTED
 * (head_dim not 64/128, rope table too large), PRSINK_ERR_LAUNCH. */
int prsink_attention(const prsink_layout* layout, const void* q, const void* k_cache,
                     const void* v_cache, void* out, float* lse, const long long* dyn_src,
                     void* stream);

/* prsink_attention with the last wave split over the key range (same result, up to float
 * rounding of the split sums).
 *
 * One CTA per SM computes a unit = (head, 256 queries).  When the units leave the last wave of
 * the device (#SM units per wave) nearly empty (384x672: 480 units = 3 waves of 148 + 36), each
 * of the r units of that wave runs as S = min(#SM / r, 8) CTAs over equal shares of the key
 * tiles; each writes its unnormalised partial (float32 O, running max, sum) to `scratch`, and
 * the last one to finish combines them (O = sum_s O_s 2^(m_s - M) / sum_s l_s 2^(m_s - M)).
 * Arguments as prsink_attention, plus:
 *   scratch        device memory of at least prsink_attention_scratch_bytes(layout) bytes,
 *                  256-byte aligned, owned by the caller, not shared with a concurrent call;
 *                  may be NULL when that size is 0 (no split planned: a plain attention)
 *   scratch_bytes  its size
 * The plan depends on the current device's SM count.  The arrival counters inside `scratch` are
 * cleared on `stream` by each call.  Errors: as prsink_attention; PRSINK_ERR_ARG for a missing,
 * misaligned or too small scratch. */
int prsink_attention_split(const prsink_layout* layout, const void* q, const void* k_cache,
                           const void* v_cache, void* out, float* lse, const long long* dyn_src,
                           void* scratch, long long scratch_bytes, void* stream);

/* prsink_attention_split without caller scratch, for callers that cannot allocate device
 * memory: an embedding runtime that owns the device's memory pool and forbids allocations
 * outside it, or a real-time loop that may not call the allocator (cudaMalloc can synchronise
 * the device and take milliseconds).  No counterpart on the pages: this is an interface for
 * such callers, not part of the method.
 *   The scratch is a file-scope device array of 20 MiB inside the library, held by every GPU
 *   that loads the library until the process exits: enough for every split plan with
 *   head_dim <= 128 on a 148-SM device (at most one partial per SM: 19.7 MB); a plan that needs
 *   more (prsink_attention_scratch_bytes, on a device with more SMs) is rejected with
 *   PRSINK_ERR_UNSUPPORTED.  The call allocates nothing (no cudaMalloc / cudaFree, no allocating
 *   library routine); it clears the array's arrival counters on `stream` before the kernel.
 *   The first call on a device looks up the array's device address with that device current;
 *   make that first call before any stream capture.  Every call shares the one array, which
 *   keeps the last call's partial results: calls that overlap on the GPU (other streams, other
 *   host threads) race on it and must be serialised by the caller.
 * Arguments, results and other errors as prsink_attention. */
int prsink_attention_split_noalloc(const prsink_layout* layout, const void* q,
                                   const void* k_cache, const void* v_cache, void* out,
                                   float* lse, const long long* dyn_src, void* stream);

/* Scratch bytes prsink_attention_split needs for `layout` on the current device (0 when the
 * last wave is full enough that no split is planned; -1 for an invalid layout). */
long long prsink_attention_scratch_bytes(const prsink_layout* layout);

/* Rotated copy of the sink keys, for prsink_attention_fused.
 *
 * [digest] weaknesses, point 2: reuse cached work to cut the repeated computation of the Ref and
 * Static Sinks.  Within a block the positions of every slot but the current block's stay fixed
 * (ring slots move one rank per block), so their keys can be rotated once per (block, layer)
 * instead of by every attention pass and every query tile.  This call rotates, for every head,
 * the raw keys of the slots in `slot_mask` (bit i = slot i) that hold data (valid_mask) at the
 * positions they have while block `layout->block_index` is generated, into k_rot.  The current
 * block's ring slot (b mod R) is never rotated (the fused attention reads that block from
 * k_new).  Rows of other slots sharing a 128-row tile with a rotated slot are rewritten with
 * their own rotation (identical for slots whose positions did not change).
 *   k_cache   bf16 [H][T][d]  raw keys (read)
 *   k_rot     bf16 [H][T][d]  rotated keys (written); a buffer of its own
 *   slot_mask slots to rotate.  A ring slot must be rotated at every block (its rank changes);
 *             ref / static / dynamic only when written (their positions never change).
 *   dyn_flag  int32 scalar or NULL: if given and 0, the dynamic slot is skipped (e.g. the
 *             retrieval's copy_out: the slot was not refilled)
 *   dyn_src   int64 scalar or NULL: if given and < 0 the dynamic slot is empty (skipped)
 * The rotation is the attention kernel's own (float32 with cos/sin tables from float64), so the
 * rotated keys equal those prsink_attention computes internally, bit for bit.
 * Errors: PRSINK_ERR_ARG, PRSINK_ERR_ALIGN, PRSINK_ERR_UNSUPPORTED, PRSINK_ERR_LAUNCH. */
int prsink_rotate_sinks(const prsink_layout* layout, const void* k_cache, void* k_rot,
                        unsigned slot_mask, const int* dyn_flag, const long long* dyn_src,
                        void* stream);

/* Attention of the current block with its Clean KV Update / per-pass append folded in.
 *
 * [digest] weaknesses, point 2 (Clean KV Update is 24.39 % of the time; cache reuse of the
 * sinks).  Equivalent to prsink_kv_append(k_new, v_new -> ring slot b mod R of k_cache /
 * v_cache) followed by prsink_attention(q, k_cache, v_cache), with the keys of every other slot
 * read already rotated from k_rot (prsink_rotate_sinks of this block, kept current by the
 * caller) instead of being rotated here.  The current block's keys are read from k_new, rotated
 * at the current block's positions and attended whatever valid_mask says about its slot; the
 * raw k_new / v_new rows are stored into the ring slot by the same launch.
 *   q, out, lse, dyn_src as prsink_attention;  k_new, v_new bf16 [L_blk][H][d] (token-major);
 *   k_rot bf16 [H][T][d] (read);  k_cache, v_cache bf16 [H][T][d]: V of the other slots read,
 *   the ring slot's K and V rows written (no other byte).
 * Errors: as prsink_attention. */
int prsink_attention_fused(const prsink_layout* layout, const void* q, const void* k_new,
                           const void* v_new, const void* k_rot, void* k_cache, void* v_cache,
                           void* out, float* lse, const long long* dyn_src, void* stream);

/* prsink_attention_fused with the last wave split over the key range (as prsink_attention_split;
 * the scratch size is prsink_attention_scratch_bytes(layout)).  Each tile of the current block is
 * still stored into the ring slot exactly once, by the share of its unit that attends it.  With
 * the heads split over several GPUs (5 of 40 heads per GPU at 8 GPUs: 55 units for 148 SMs)
 * every unit runs as two shares.  Arguments as prsink_attention_fused plus scratch /
 * scratch_bytes as prsink_attention_split.  Errors: as those two calls. */
int prsink_attention_fused_split(const prsink_layout* layout, const void* q, const void* k_new,
                                 const void* v_new, const void* k_rot, void* k_cache,
                                 void* v_cache, void* out, float* lse, const long long* dyn_src,
                                 void* scratch, long long scratch_bytes, void* stream);

/* Clean KV Update / per-pass append: write one slot's raw K and V into the caches.
 *
 * [digest] pipeline, inference clause: KV_cache <- KV_cache U Forward(z^0_b, t=0, C) is
 * written into the rolling window, keys raw (pre-RoPE); the ring slot of block b is b mod R;
 * block 0's clean K/V also fills the static sink ([abstract]).
 *
 *   k_new, v_new  bf16 [n][H][d] token-major (as a QKV projection emits them), n = the slot's
 *                 row count (L_ref for the ref slot, L_blk otherwise)
 *   k_cache, v_cache  bf16 [H][T][d]; rows of slot `dest_slot` are overwritten, no other byte
 *   dest_slot     PRSINK_SLOT_REF / _STATIC / _DYNAMIC or PRSINK_SLOT_RING0 + s
 * Bit copy (no rounding).  Errors: PRSINK_ERR_ARG, PRSINK_ERR_ALIGN, PRSINK_ERR_LAUNCH. */
int prsink_kv_append(const prsink_layout* layout, const void* k_new, const void* v_new,
                     void* k_cache, void* v_cache, int dest_slot, void* stream);

/* 558-d pose fingerprint of one block.
 *
 * [digest] pipeline, inference clause: 62 keypoints x 3 frames x 3 values, l2-normalised;
 * [digest] novelty, point 2: confidence channel included, failed frames zero-filled.
 *   kp        f32 [3][62][3] (x, y, conf) per frame, flattened in that order
 *   frame_ok  u8  [3], 0 = detection failed (the frame contributes zeros)
 *   phi       f32 [558] (written); an all-zero vector is written as zeros
 * Norm accumulated in float64.  Errors: PRSINK_ERR_ARG, PRSINK_ERR_LAUNCH. */
int prsink_fingerprint(const float* kp, const unsigned char* frame_ok, float* phi, void* stream);

/* Pose retrieval r(b) = argmax_i phi_b . phi_i over the bank, excluding the entry of block
 * b-1 (already in the window), and the copy of that entry's K/V into the dynamic sink.
 *
 * [digest] pipeline, inference clause: retrieve before generating the block, excluding b-1,
 * copy the entry's KV into the Dynamic Sink; [digest] novelty, point 2: cosine maximisation
 * as one dot product over l2-normalised fingerprints.
 *
 *   phi_b       f32 [558]          fingerprint of the incoming block
 *   bank_phi    f32 [M][558]       bank fingerprints
 *   bank_src    int64 [M]          source block of each entry
 *   bank_count  int32 scalar       entries in use (0..M), slots 0..count-1
 *   M           bank capacity (1..PRSINK_MAX_BANK)
 *   exclude_block  b-1 (entries with this source are not eligible)
 *   r_out       int32 scalar (written): chosen slot, ties to the lowest slot, -1 if none
 *   score_out   f32 scalar (written) or NULL: the chosen similarity (-inf if none)
 *   copy_out    int32 scalar (written): 1 if the dynamic sink must be (re)filled from entry
 *               r, i.e. r >= 0 and bank_src[r] differs from the incoming *dyn_src; else 0
 *   dyn_src     int64 scalar, in/out: source block held by the dynamic sink (-1 = empty).
 *               On return it is bank_src[r] (or -1 when r = -1).
 *   bank_kv, cache_kv, n_layers: optional (all NULL/0 to skip the copy).  When given, the
 *               dynamic slot of every layer is overwritten with bank entry r iff *copy_out.
 *               The copy addresses bank_kv as bf16 [n_layers][M][2][H][L_blk][d] and cache_kv
 *               as bf16 [n_layers][2][H][T][d] (H, d, L_blk, T from `layout`): the caller must
 *               pass buffers of exactly these sizes (the library cannot check device sizes;
 *               the Python binding does).
 * Similarities are accumulated in float64.  Errors: PRSINK_ERR_ARG, _ALIGN, _LAUNCH. */
int prsink_retrieve(const prsink_layout* layout, const float* phi_b, const float* bank_phi,
                    const long long* bank_src, const int* bank_count, int M,
                    long long exclude_block, int* r_out, float* score_out, int* copy_out,
                    long long* dyn_src, const void* bank_kv, void* cache_kv, int n_layers,
                    void* stream);

/* Diversity-driven memory-bank update after block b's Clean KV Update.
 *
 * [digest] novelty, point 3: exhaustive replacement minimising the mean intra-bank
 * similarity (write for coverage, read for relevance); [digest] weaknesses, point 3 and
 * reproducibility: M = 5, written during the first 20 blocks, then frozen.
 * For b >= write_blocks nothing changes (action -1).  While count < M the block is inserted
 * at slot count.  Otherwise the options "keep" and "replace slot j" are scored by the mean
 * of phi_i . phi_j over unordered pairs of the resulting bank (float64); the least wins,
 * ties go to keep, then to the lowest j.
 *
 *   bank_phi   f32 [M][558]  in/out      bank_src  int64 [M] in/out      bank_count int32 in/out
 *   phi_b      f32 [558]     fingerprint of block b
 *   action_out int32 scalar (written): slot written, or -1
 *   cache_kv, bank_kv, n_layers: optional (NULL/0 to skip).  When given and action >= 0, the
 *               clean K/V of block b (ring slot b mod R of every layer) is copied into bank
 *               entry `action`.  Sizes as for prsink_retrieve: bank_kv bf16
 *               [n_layers][M][2][H][L_blk][d], cache_kv bf16 [n_layers][2][H][T][d].
 * Errors: PRSINK_ERR_ARG, PRSINK_ERR_ALIGN, PRSINK_ERR_LAUNCH. */
int prsink_bank_update(const prsink_layout* layout, float* bank_phi, long long* bank_src,
                       int* bank_count, int M, const float* phi_b, long long b,
                       int write_blocks, int* action_out, const void* cache_kv, void* bank_kv,
                       int n_layers, void* stream);

/* ---- bank policy variants -------------------------------------------------------------
 * [digest] weaknesses, point 3: a bank frozen after the first 20 blocks assumes the pose
 * distribution is sampled at the start of the stream; proposed fixes are continuous writes
 * with decaying weights and a refresh gated on fingerprint distance.  [digest] weaknesses,
 * point 5: under failed detection retrieval degrades; a proposed fix is to fall back to the
 * conservative Static Sink + window cache.  These calls implement those readings; the calls
 * above implement the pages' own rule. */
#define PRSINK_BANK_FROZEN 0       /* the pages' rule: diversity writes, then frozen        */
#define PRSINK_BANK_DECAY  1       /* after the freeze: moving average into the nearest entry */
#define PRSINK_BANK_GATED  2       /* after the freeze: diversity rule for far-away blocks   */

#define PRSINK_BANK_MODE_NONE  0   /* mode word: nothing written                            */
#define PRSINK_BANK_MODE_STORE 1   /* the block's fingerprint and K/V replace entry `action` */
#define PRSINK_BANK_MODE_BLEND 2   /* entry `action` averaged with the block                */

typedef struct prsink_bank_policy {
  int kind;            /* PRSINK_BANK_FROZEN / _DECAY / _GATED                               */
  int write_blocks;    /* the diversity rule runs for blocks b < write_blocks (20)           */
  float alpha;         /* DECAY, in [0, 1]: weight of the block.  For b >= write_blocks the
                          block goes into its nearest entry j = argmax_i phi_b . phi_i (ties
                          to the lowest slot): phi_j <- l2-normalised((1-alpha) phi_j + alpha
                          phi_b) (float64), every K/V element x of entry j (all layers) <-
                          bf16(fl32(fl32(w_old x) + fl32(alpha z))), w_old = fl32(1 - alpha),
                          z the block's clean K/V; src_j <- b.  alpha = 0 writes nothing.    */
  float gate;          /* GATED: for b >= write_blocks the diversity rule runs for a block
                          with min_i ||phi_b - phi_i||_2 > gate (float64), else nothing is
                          written                                                            */
} prsink_bank_policy;

/* prsink_retrieve with the fallback to Static Sink + window: when fewer than `min_detected`
 * (0..3) of the block's frames were detected (frame_ok: u8 [3] on the device, as given to
 * prsink_fingerprint), no entry is retrieved: r = -1, *dyn_src = -1 (the dynamic sink is empty
 * for the block's attention calls), *copy_out = 0.  Otherwise identical to prsink_retrieve.
 * Errors: as prsink_retrieve; PRSINK_ERR_ARG for a null frame_ok or min_detected outside
 * [0, 3]. */
int prsink_retrieve_fallback(const prsink_layout* layout, const float* phi_b,
                             const unsigned char* frame_ok, int min_detected,
                             const float* bank_phi, const long long* bank_src,
                             const int* bank_count, int M, long long exclude_block, int* r_out,
                             float* score_out, int* copy_out, long long* dyn_src,
                             const void* bank_kv, void* cache_kv, int n_layers, void* stream);

/* prsink_bank_update under a policy.  For b < policy->write_blocks, and for every block with
 * PRSINK_BANK_FROZEN, identical to prsink_bank_update with write_blocks = policy->write_blocks.
 *   action_out  int32 scalar (written): the entry written, or -1
 *   mode_out    int32 scalar (written, device, required): PRSINK_BANK_MODE_*; the K/V copies
 *               that follow read it, so the decision stays on the device
 *   cache_kv, bank_kv, n_layers: as prsink_bank_update; a store copies block b's clean K/V
 *               (ring slot b mod R of every layer) into entry `action`, a blend averages it in.
 * Errors: as prsink_bank_update; PRSINK_ERR_ARG for a null policy or mode_out, an unknown kind,
 * alpha outside [0, 1], a non-finite gate or write_blocks < 0. */
int prsink_bank_update_policy(const prsink_layout* layout, const prsink_bank_policy* policy,
                              float* bank_phi, long long* bank_src, int* bank_count, int M,
                              const float* phi_b, long long b, int* action_out, int* mode_out,
                              const void* cache_kv, void* bank_kv, int n_layers, void* stream);

/* Synchronise `stream`, then read and clear the status word of the current device:
 * PRSINK_OK, or PRSINK_ERR_TIMEOUT if a bounded wait of any kernel on this device (any
 * stream) ran out since the word was last cleared, or PRSINK_ERR_LAUNCH.  Only `stream` is
 * synchronised: kernels still running on other streams may report later. */
int prsink_sync_status(void* stream);

/* Text of the last host-side error of this thread ("" if none).  Owned by the library. */
const char* prsink_last_error(void);

/* Number of kernels this library launched since load (host counter). */
long long prsink_launch_count(void);

/* Self-test of the bounded-wait path: launches one block that waits on a barrier nothing
 * signals, gives up after `timeout_ns` (clamped to [1e3, 5e9] ns), records
 * PRSINK_ERR_TIMEOUT in the status word and returns.  No GPU fault, no hang. */
int prsink_debug_wait_timeout(long long timeout_ns, void* stream);

/* Self-test of the attention kernel's own abort path.  Arms the next prsink_attention /
 * prsink_attention_fused / prsink_rotate_sinks call of this host thread (one call only): its
 * bounded waits give up after `timeout_ns` (clamped to [1e4, 1e9] ns) instead of 2 s, and in an
 * attention call the MMA issuer withholds the first commit of query tile 0, so that the softmax
 * wait runs out.  The kernel then raises its abort flag, records PRSINK_ERR_TIMEOUT in the status
 * word, lets its copies and MMAs in flight complete, frees its tensor memory and writes out = 0,
 * lse = -inf for the rows it did not finish.  No GPU fault, no hang; the next call is normal. */
int prsink_debug_attention_stall(long long timeout_ns);

/* Library ABI version (increments on any signature change). */
int prsink_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PRSINK_H */
