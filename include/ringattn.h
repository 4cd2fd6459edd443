/*
 * ringattn.h -- C ABI of the B200 (sm_100a) exact blockwise attention library
 * (libringattn.so).
 *
 * The library computes exact causal (or full) softmax attention the way Ring
 * Attention and Striped Attention organise it: the sequence is split into P
 * virtual shards; each shard's query block stays put while the key/value
 * blocks visit it in ring order, one block per round, and every round is
 * folded in with an online softmax (running max m, running normaliser l,
 * output rescaled when m grows).  Fully masked tiles are skipped.
 *
 * Sources for the operations (page title, section):
 *   - "ICLR 2024論文解説: Ring Attention -- 複数GPU間でのブロックワイズ分散
 *     アテンションによる超長コンテキスト処理": ステップ1 (contiguous split),
 *     ステップ2 (ring rounds), ステップ3 (online-softmax recurrence; scores
 *     scaled by 1/sqrt(d)), 実装例 (unnormalised accumulator, one final
 *     division by the row sum).
 *   - "Striped Attention: Faster Ring Attention for Causal Transformers"
 *     (paper review): 核心公式 (CausalAttn = Softmax(QK^T + C)V), 分区策略对比
 *     (token t on device t mod P), GetMask 函数 (block masks), 分块与分瓦片
 *     (skip fully masked tiles), 位置编码处理 (position ids striped alike).
 *   - 1cademy, "Computing Attention Weights in Sequence Parallelism": the
 *     softmax denominator as a sum of per-node partial sums (lse merge, the
 *     per-round partials of the ring).
 *   - aiunderstanding.org, "Parallélisme de séquence et attention en
 *     anneau": L'avenir (zigzag named as a causal rebalancing variant beside
 *     striping; the layout's definition here is a reading, see RA_ZIGZAG).
 *
 * Conventions for every entry point:
 *   - All pointers marked "device" are CUDA device pointers on the current
 *     device; the caller allocates and owns every buffer (including the
 *     backward's workspace and ra_attn_fwd_host's staging workspace).  The
 *     library never allocates device memory at run time (its only device
 *     data are static: a 4-byte fault word and ra_attn_bwd_noalloc's 4 MiB
 *     scratch) and keeps no pointer after a call returns.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL =
 *     the legacy default stream).  A return of RA_OK means the work was
 *     validated and enqueued, not that it finished.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns a non-zero status and launches nothing.  No entry
 *     point aborts, prints, or traps on the device.
 *   - Tensors are dense row-major.  [B, H, N, d] bf16 means element
 *     (b, h, n, i) at ((b*H + h)*N + n)*d + i, two bytes each.
 *   - Thread safety: calls may be made from several host threads.  The
 *     exceptions share library state: ra_attn_bwd_noalloc's scratch (calls
 *     must not overlap on the GPU) and ra_attn_fwd_host's copy streams
 *     (calls on one device are enqueued one at a time).
 *   - Per device the library looks up, once, the device addresses of its
 *     static data (and creates ra_attn_fwd_host's copy streams); it keeps
 *     them until the process exits, so it must not be used on a device
 *     after a cudaDeviceReset of that device.
 */
#ifndef RINGATTN_H_
#define RINGATTN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int ra_status;

/* Status codes. */
#define RA_OK 0
#define RA_ERR_NULL 1        /* a required pointer is NULL                     */
#define RA_ERR_ALIGN 2       /* a pointer is not 16-byte aligned               */
#define RA_ERR_SHAPE 3       /* sizes out of range, or N not a multiple of P   */
#define RA_ERR_HEADDIM 4     /* head dimension d not supported (64 or 128)     */
#define RA_ERR_LAYOUT 5      /* unknown layout / flag bits                     */
#define RA_ERR_SCALE 6       /* scale not finite or not > 0                    */
#define RA_ERR_DTYPE 7       /* unknown dtype code                             */
#define RA_ERR_ALIAS 8       /* input and output buffers overlap               */
#define RA_ERR_CUDA 9        /* a CUDA runtime/driver call failed              */
#define RA_ERR_DEVICE 10     /* current device is not sm_100 (B200)            */
#define RA_ERR_DEVICE_FAULT 11 /* a kernel gave up a bounded wait (see below)  */
#define RA_ERR_SCRATCH 12    /* problem larger than the built-in scratch of    */
                             /* ra_attn_bwd_noalloc (B*H*N > 1048576)          */
#define RA_ERR_ROPE 13       /* unknown RoPE pairing, or base not > 1 / finite */
#define RA_ERR_WORKSPACE 14  /* device workspace too small                     */
#define RA_ERR_NOPROFILE 15  /* library built without the phase profile        */

/* Layouts (low byte of `layout`). */
#define RA_CONTIGUOUS 0      /* shard j = tokens [j*c, (j+1)*c)  (Ring)        */
#define RA_STRIPED 1         /* shard j = tokens j, j+P, j+2P, ...  (Striped)  */
#define RA_ZIGZAG 2          /* shard j = chunks j and 2P-1-j of 2P chunks      */
                             /* (a reading: the pages only name "zigzag";      */
                             /* needs N/P even; attention needs N/P % 512 == 0; */
                             /* not for ra_attn_fwd_block / ra_tile_census)     */

/* Optional scheduling flag for ra_attn_fwd, OR-ed into `layout`.
 * Default ("owner" schedule): each virtual shard j is served by its own fixed
 * group of floor(#SM / P) streaming multiprocessors, which walk that shard's
 * query tiles through all P rounds -- the per-device work of the ring, so
 * the wall time is set by the most loaded shard as on P real devices.
 * RA_SCHED_FREE: every SM takes work from every shard (a single-GPU
 * load-balanced schedule; same results, same tile skipping). */
#define RA_SCHED_FREE 0x100

/* Optional kernel flag for ra_attn_fwd, OR-ed into `layout`: RA_CTA_PAIR
 * runs the forward on pairs of SMs (clusters of two CTAs sharing each
 * tensor-core MMA, M = 256; each SM loads half of every key/value tile).
 * It applies to d = 128 in layout order (not RA_TOKEN_ORDER, not RA_ZIGZAG);
 * elsewhere it is ignored.  Same results (bit-identical on the shapes
 * tested): each row is the same online softmax over the same key tiles.
 * On B200 it measured slower than the default kernel at every benchmark
 * shape (717 against 1023 TFLOP/s at N = 131072, H = 8, P = 8 striped): the
 * MMA issuer waits for the softmax of both SMs, across the pair, on every
 * tile.  Not recommended for speed; it exists as the tested two-SM form. */
#define RA_CTA_PAIR 0x800

/* Optional output flag for ra_attn_fwd, OR-ed into `layout`: O is written as
 * float32 [B, H, N, d] (o must hold 4 bytes per element) instead of bf16,
 * e.g. for callers that merge partial results or want O before rounding. */
#define RA_O_F32 0x200

/* Optional flag for ra_attn_fwd and ra_attn_bwd, OR-ed into `layout`: all
 * their tensors (q, k, v, o, lse; dO and the gradients) are in TOKEN order.
 * The layout's permutation is then applied inside the kernel (the TMA loads
 * address shard j's rows where the tokens live, the epilogue writes each row
 * to its token position), so no ra_partition pass is needed before or after;
 * results equal the partition / attention / inverse-partition sequence bit
 * for bit. */
#define RA_TOKEN_ORDER 0x400

/* Rotation pairs of ra_partition_rope. */
#define RA_ROPE_INTERLEAVED 0 /* pair i = dimensions (2i, 2i+1)                */
#define RA_ROPE_HALF 1        /* pair i = dimensions (i, i + d/2)              */

/* Element types for ra_partition. */
#define RA_BF16 0
#define RA_F32 1
#define RA_I32 2

/* Human-readable text for a status code (static storage; never NULL). */
const char* ra_status_string(ra_status status);

/* Library version, as major*10000 + minor*100 + patch. */
int ra_version(void);

/*
 * ra_partition -- move rows between token order and layout order.
 *
 * Defined by the placements of "Striped Attention" review 分区策略对比 and
 * Ring Attention explainer ステップ1: with c = N/P, layout slot s = j*c + x
 * (shard j, local index x) holds token t = x*P + j (RA_STRIPED),
 * t = j*c + x (RA_CONTIGUOUS), or, with h = c/2, t = j*h + x for x < h and
 * t = (2P-1-j)*h + (x - h) otherwise (RA_ZIGZAG, a reading of the layout the
 * pages only name).  Position ids are moved the same way
 * (Striped review, 位置编码处理): pass the int32 ids as [1, 1, N, 1] RA_I32.
 *
 *   src, dst  device, [B, H, N, d] of `dtype` (bf16 = 2 bytes, f32/i32 = 4).
 *             Must not overlap (RA_ERR_ALIAS); 16-byte aligned when a row
 *             (d * element size) is a multiple of 16 bytes, else 4-byte
 *             aligned.
 *   inverse   0: token order -> layout order  (dst[.,.,s,:] = src[.,.,t(s),:])
 *             1: layout order -> token order  (dst[.,.,t(s),:] = src[.,.,s,:])
 *   P         number of shards, 1 <= P <= N, N % P == 0.
 *   d         row length in elements (any value >= 1; use d = 1 for lse or
 *             position ids); d * element size < 2^30.
 *   B, H, N   >= 1 with B*H*N < 2^31 (else RA_ERR_SHAPE).
 * The result is a pure byte permutation (bit-exact).  RA_CONTIGUOUS is the
 * identity and is performed as a copy.
 */
ra_status ra_partition(const void* src, void* dst, int64_t B, int64_t H, int64_t N, int64_t d,
                       int P, int layout, int inverse, int dtype, void* stream);

/*
 * ra_partition_rope -- token order -> layout order with rotary position
 * embedding applied at the ORIGINAL token positions.
 *
 * The Striped review (位置编码处理) requires a position encoding such as RoPE
 * to see the same stripe permutation as the tokens.  The pages name RoPE but
 * do not define it; this is RoFormer's rotation: with theta_i =
 * base^(-2i/d), pair i of row t is turned by the angle t * theta_i,
 *     (u, w) -> (u cos - w sin, u sin + w cos),
 * the pair being dimensions (2i, 2i+1) (RA_ROPE_INTERLEAVED) or (i, i + d/2)
 * (RA_ROPE_HALF).  dst[b,h,s,:] = RoPE(src[b,h,t(s),:], t(s)), with t(s) the
 * token held by layout slot s (as ra_partition, inverse = 0).  Apply it to q
 * and k; v goes through ra_partition.  The same result as striping the
 * position ids first and rotating in layout order.
 *
 *   src, dst  device bf16 [B, H, N, d], 16-byte aligned, not overlapping
 *             (RA_ERR_ALIAS).
 *   d         a multiple of 16, 16 <= d <= 512 (else RA_ERR_HEADDIM).
 *   B, H, N, P  as ra_partition (B*H*N < 2^31, N % P == 0).
 *   base      RoPE base (e.g. 10000), finite and > 1 (else RA_ERR_ROPE).
 *   pairing   RA_ROPE_INTERLEAVED or RA_ROPE_HALF (else RA_ERR_ROPE).
 * Angles are evaluated in double precision, the rotation in fp32, and the
 * result is rounded to bf16 once (within one bf16 rounding of the exact
 * value).  RA_CONTIGUOUS applies the rotation without moving rows.
 */
ra_status ra_partition_rope(const void* src, void* dst, int64_t B, int64_t H, int64_t N,
                            int64_t d, int P, int layout, int pairing, float base, void* stream);

/*
 * ra_attn_fwd -- exact blockwise attention forward over P virtual shards.
 *
 * Computes, per (b, h), O = Softmax(Q K^T * scale + C) V and
 * lse[i] = ln sum_t exp(Q_i . K_t * scale + C_it) (natural log), where C is
 * -inf where the key's ORIGINAL token index exceeds the query's (causal != 0)
 * and 0 otherwise (Striped review 核心公式; Ring explainer ステップ3).  The
 * shard loop follows the ring: shard j's query tiles meet key block
 * (j - r) mod P in round r, folded in with online softmax; tiles that the
 * layout's GetMask hides completely are not computed.
 *
 *   q, k, v  device, [B, H, N, d] bf16, rows already in LAYOUT order (see
 *            ra_partition), 16-byte aligned.
 *   o        device, [B, H, N, d] bf16 output (float32 with RA_O_F32),
 *            layout order, 16-byte aligned.  Must not overlap q, k, v.
 *   lse      device, [B, H, N] float32 output, layout order, 16-byte aligned.
 *   d        64 or 128.
 *   N, P     1 <= P, N % P == 0, c = N / P <= 2^30 / 128; any c (a ragged
 *            last tile of a shard is masked).  B*H*N < 2^31.
 *   layout   RA_CONTIGUOUS, RA_STRIPED or RA_ZIGZAG (N/P a multiple of
 *            512), optionally | RA_SCHED_FREE, | RA_O_F32, | RA_TOKEN_ORDER
 *            (then q, k, v, o, lse are in token order).
 *   causal   0: no mask (the layout then only permutes rows); else causal in
 *            original token order.
 *   scale    > 0 and finite; 1/sqrt(d) is the usual value.
 * Arithmetic: bf16 operands, fp32 accumulation of Q K^T and P V on the
 * tensor cores, fp32 softmax statistics, probabilities rounded to bf16 for
 * the P V product, O rounded to bf16 once at the end (not with RA_O_F32).
 */
ra_status ra_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                      int64_t B, int64_t H, int64_t N, int64_t d, int P, int layout,
                      int causal, float scale, void* stream);

/*
 * ra_attn_bwd -- gradients of ra_attn_fwd: dQ, dK, dV.
 *
 * The pages give no backward algorithm (the Striped review measures training
 * speedups, 五 核心结果); this is the derivative of the forward's definition
 * (Striped review 核心公式) over the same shards, masks and skipped tiles:
 *   P = exp(Q K^T * scale + C - lse),  D = rowsum(dO o O),
 *   dS = P o (dO V^T - D),  dV = P^T dO,  dK = dS^T Q * scale,  dQ = dS K * scale.
 *
 *   q, k, v, o, dout  device, [B, H, N, d] bf16, layout order (o and lse as
 *                     returned by ra_attn_fwd on the same q, k, v).
 *   lse               device, [B, H, N] float32, layout order.
 *   dq, dk, dv        device, [B, H, N, d] bf16 outputs, layout order; must
 *                     not overlap each other or any input.
 *   workspace         device, float32[B * H * N] scratch the call overwrites
 *                     (holds D); owned by the caller, no overlap with others.
 *   All pointers 16-byte aligned.  d, N, P, layout, causal and scale as for
 *   ra_attn_fwd; of the flags only RA_TOKEN_ORDER (every tensor, lse
 *   included, in token order).
 * Arithmetic: bf16 operands, fp32 accumulation on the tensor cores, P and dS
 * rounded to bf16 for their products, outputs rounded to bf16 once.
 */
ra_status ra_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                      float* workspace, int64_t B, int64_t H, int64_t N, int64_t d, int P,
                      int layout, int causal, float scale, void* stream);

/*
 * ra_attn_bwd_noalloc -- ra_attn_bwd for callers that cannot allocate.
 *
 * No counterpart in the paper: this is a library convenience.  Some callers
 * are handed their input and output buffers by a host framework that owns
 * all device memory (a plug-in, an embedded runtime, a serving process with
 * a fixed memory budget) and may not allocate more, or cannot afford a
 * device allocation that might block or fail in the middle of a step.  For
 * them this entry point takes no workspace: the backward's scratch row
 * vector (D, one float per query row) lives in a fixed array inside the
 * library, 2^20 floats (4 MiB) reserved on every GPU that loads the library
 * until the process exits.  It calls no allocator.
 *
 *   Arguments as for ra_attn_bwd, minus `workspace`.
 *   B * H * N must be <= 1048576, else RA_ERR_SCRATCH (nothing launched).
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   All calls on one device share that device's array: calls whose kernels
 *   overlap on the same GPU race on it and give wrong results; order them on
 *   one stream.  The looked-up address is kept for the life of the process:
 *   do not use the library across a cudaDeviceReset of that device.
 */
ra_status ra_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              int64_t B, int64_t H, int64_t N, int64_t d, int P, int layout,
                              int causal, float scale, void* stream);

/*
 * ra_attn_fwd_host -- the whole forward path from host memory: token-order
 * q, k, v in host memory -> (partition, attention, un-partition) -> token-
 * order o, lse in host memory.
 *
 * Same computation and results as ra_partition + ra_attn_fwd + ra_partition
 * (inverse) on device copies (bit-identical: every (b, h) is computed alone).
 * The heads are processed in chunks through two staging slots of the
 * caller's device workspace (each chunk runs the attention with
 * RA_TOKEN_ORDER, so only q, k, v, o, lse are staged): the host-to-device
 * copy of chunk i+1 and the device-to-host copy of chunk i-1 run on the
 * library's own copy streams while chunk i computes on `stream`.  The first
 * and last chunks take half as many heads as the others (their copies in
 * and out overlap no compute).  Host buffers should be page-locked (pinned)
 * for the copies to overlap.
 *
 *   q, k, v     host bf16 [B, H, N, d], token order.
 *   o, lse      host bf16 [B, H, N, d] and float32 [B, H, N], token order.
 *   workspace   device buffer, 256-byte aligned, of workspace_bytes >=
 *               ra_attn_fwd_host_workspace(N, d, layout, 1) (else
 *               RA_ERR_WORKSPACE); more allows larger chunks (up to a
 *               quarter of the heads each).
 *   other arguments and errors as ra_attn_fwd.
 * Stream-ordered: work on `stream` after this call sees o and lse written.
 * The library allocates nothing; its two copy streams and a few events are
 * created on the first call on a device (make that call before any stream
 * capture).  Calls on one device are enqueued one at a time; two calls that
 * share a workspace must be ordered on one stream.
 */
ra_status ra_attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                           int64_t B, int64_t H, int64_t N, int64_t d, int P, int layout,
                           int causal, float scale, void* workspace, int64_t workspace_bytes,
                           void* stream);

/* Device workspace bytes for ra_attn_fwd_host with `heads_per_chunk` heads
 * per chunk (two staging slots); -1 for invalid sizes (N outside
 * [1, 2^31), d outside [1, 1024], heads_per_chunk < 1, or a byte count that
 * does not fit int64_t). */
int64_t ra_attn_fwd_host_workspace(int64_t N, int64_t d, int layout, int64_t heads_per_chunk);

/*
 * ra_attn_fwd_block -- one round of one device of the ring: query shard j
 * against key/value block kb, normalised over that block alone.
 *
 * The physical ring (Ring explainer ステップ2 and its 実装例: each device keeps
 * its Q block, sends its K/V block to rank+1 and receives from rank-1, so in
 * round r device j holds block (j - r) mod P) computes, every round, the
 * attention of its query block against the block it holds, and the rounds
 * are combined through their softmax normalisers (1cademy page "Computing
 * Attention Weights in Sequence Parallelism": the denominator is a sum of
 * per-node partial sums).  This is that per-round computation with the
 * GetMask of the pair (j, kb) (Striped review, GetMask 函数); combine rounds
 * with ra_lse_merge_acc.
 *
 *   q         device bf16 [B, H, c, d]: query shard j in layout order.
 *   k, v      device bf16 [B, H, c, d]: key/value block kb in layout order.
 *   o, lse    outputs: bf16 [B, H, c, d] (float32 with RA_O_F32 OR-ed into
 *             layout) and float32 [B, H, c].  A query row that sees no key
 *             of the block gets o = 0, lse = -inf.
 *   j, kb, P  0 <= j, kb < P: the pair's shard indices (masks only).
 *   d         64 or 128; c = N / P >= 1.
 *   layout    RA_CONTIGUOUS or RA_STRIPED, optionally | RA_O_F32.  A ring
 *             that keeps its per-round partials in float32 (RA_O_F32 here,
 *             RA_MERGE_F32_PARTIAL in ra_lse_merge_acc) rounds O to bf16
 *             once, at the end; bf16 partials add one more rounding per
 *             row, which a peaked softmax (one dominant key) does not
 *             average away.
 * Same tile skipping and precision as ra_attn_fwd.  Errors as ra_attn_fwd.
 */
ra_status ra_attn_fwd_block(const void* q, const void* k, const void* v, void* o, float* lse,
                            int64_t B, int64_t H, int64_t c, int64_t d, int j, int kb, int P,
                            int layout, int causal, float scale, void* stream);

/* Modes of ra_lse_merge_acc (OR-ed). */
#define RA_MERGE_FIRST 1     /* accumulator not yet set: it becomes the partial */
#define RA_MERGE_FINAL 2     /* also write the merged O as bf16 to o_final      */
#define RA_MERGE_F32_PARTIAL 4 /* the partial o_b is float32, not bf16          */

/*
 * ra_lse_merge_acc -- fold a partial result into a float32 accumulator (the
 * same merge as ra_lse_merge; 1cademy page "Computing Attention Weights in
 * Sequence Parallelism"), so that P rounds round to bf16 once.
 *
 *   o_acc, lse_acc   device float32 [rows, d] and [rows], read and written.
 *   o_b, lse_b       device bf16 [rows, d] (float32 with
 *                    RA_MERGE_F32_PARTIAL) and float32 [rows]: the partial.
 *   o_final          device bf16 [rows, d], written when mode has
 *                    RA_MERGE_FINAL (may be NULL otherwise).
 *   rows, d          0 <= rows < 2^31; d a multiple of 8, 8 <= d <= 2^20
 *                    (else RA_ERR_SHAPE).
 * No buffer may overlap another (RA_ERR_ALIAS); o_acc, o_b, o_final 16-byte
 * aligned.  Unknown mode bits: RA_ERR_LAYOUT.  Empty sides (lse = -inf)
 * contribute nothing; both empty give o = 0, lse = -inf.
 */
ra_status ra_lse_merge_acc(float* o_acc, float* lse_acc, const void* o_b, const float* lse_b,
                           void* o_final, int64_t rows, int64_t d, int mode, void* stream);

/*
 * ra_lse_merge -- merge two partial attention results over disjoint key sets.
 *
 * From the split of the softmax denominator into per-node partial sums
 * (1cademy, "Computing Attention Weights in Sequence Parallelism"):
 *   lse = ln(e^lse_a + e^lse_b);  o = e^(lse_a - lse) o_a + e^(lse_b - lse) o_b
 * A side with lse = -inf contributes nothing; both -inf gives o = 0,
 * lse = -inf.
 *
 *   o_a, o_b, o_out      device, [rows, d] bf16, 16-byte aligned.
 *   lse_a, lse_b, lse_out device, [rows] float32.
 *   o_out may alias o_a (and lse_out lse_a): each element is read before it
 *   is written by the same thread.
 *   0 <= rows < 2^40 (0 is a no-op); d % 8 == 0, 8 <= d <= 2^20 (else
 *   RA_ERR_SHAPE).
 * Arithmetic in fp32, o_out rounded to bf16.
 */
ra_status ra_lse_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                       void* o_out, float* lse_out, int64_t rows, int64_t d, void* stream);

/*
 * ra_tile_census -- count, on the device, what ra_attn_fwd's schedule does.
 *
 * For every query shard j and round r (key block (j - r) mod P), counts with
 * the attention kernel's own tile classifier and per-row mask limits:
 *   out[(j*P + r)*4 + 0]  tiles skipped
 *   out[(j*P + r)*4 + 1]  tiles computed without a mask
 *   out[(j*P + r)*4 + 2]  tiles computed with a per-element mask
 *   out[(j*P + r)*4 + 3]  visible (query, key) pairs = the round's work
 * for one (b, h) (every head has the same schedule).  Tiles are 128 x 128.
 * The visible-pair counts are the per-device, per-round work of the Striped
 * review (Ring Attention 工作负载 / Striped Attention 工作负载).
 *
 *   out   device, int64[P * P * 4], 8-byte aligned; overwritten.
 *   N, P  as for ra_attn_fwd (d plays no role).
 */
ra_status ra_tile_census(int64_t N, int P, int layout, int causal, int64_t* out, void* stream);

/*
 * ra_device_fault -- read and clear the library's device fault word.
 *
 * Every wait inside the library's kernels is bounded.  A kernel that gives up
 * a wait records a non-zero code here, releases what it holds and returns
 * early (its outputs are then incomplete).  This call synchronises the
 * current device, stores the word in *code (0 = no fault) and clears it.
 * Returns RA_ERR_DEVICE_FAULT if the word was non-zero, RA_OK otherwise.
 */
ra_status ra_device_fault(int* code);

/*
 * ra_fwd_phase_profile -- read and clear the forward kernel's phase counters.
 *
 * Not an operation of the pages: a diagnostic of where the attention kernel
 * spends its cycles.  Only a library built with RA_PROFILE=1 (`python -m
 * long_context_exact_attn_b200.build --profile` writes libringattn_prof.so)
 * keeps counters; the regular library returns RA_ERR_NOPROFILE.  In the
 * profiling build every ra_attn_fwd launch adds, for each of its first 160
 * CTAs, the clock64 cycles that each softmax warp (slots 0-7) and the MMA
 * warp (slot 8) spent in each phase of its loop; slot 9 is unused.  Softmax
 * phases: 0 loop, skipped tiles and epilogue, 1 waiting for S, 2 loading S
 * from tensor memory, 3 row max and rescale decision, 4 exps of the first
 * part of P (keys 0-63; 0-95 when the work-list schedule of small striped
 * problems runs) with the O rescale and the first publication of P, 5 exps
 * of the rest and the last publication, 6 unused, 7 tiles processed.  MMA
 * phases: 0 issuing, 1 waiting for the next K tile, 2 for the V tile, 3 for
 * the first part of P, 4 for the rest, 5 for a released O (epilogue), 6
 * unused, 7 key-tile steps.  The timers themselves cost a few per cent.
 * This call synchronises the current device, copies the counters to
 * host memory as uint64 [160][10][8] and clears them.
 *
 *   out       host array of at least 160 * 10 * 8 = 12800 uint64 values.
 *   capacity  its length; smaller: RA_ERR_SHAPE.
 */
ra_status ra_fwd_phase_profile(uint64_t* out, int64_t capacity);

/*
 * ra_wait_selftest -- exercise the bounded-wait and fault-reporting path.
 *
 * Not an operation of the pages: a diagnostic for the library's failure
 * detection.  Launches one warp that waits, through the same bounded wait
 * the attention kernel uses, on a barrier that nothing ever completes.  The
 * wait gives up after limit_ns nanoseconds of wall time; the kernel then
 * records fault code 2 in the device fault word and returns, leaving the
 * CUDA context usable.  Read the code with ra_device_fault().
 *
 *   limit_ns  1000 <= limit_ns <= 1e10, else RA_ERR_SHAPE.
 */
ra_status ra_wait_selftest(int64_t limit_ns, void* stream);

/*
 * ra_attn_abort_selftest -- exercise the attention kernel's own abort path.
 *
 * Not an operation of the pages: a diagnostic for the library's failure
 * detection.  Runs ra_attn_fwd on the given arguments (same meaning, layout,
 * ownership and validation) with one change: in every CTA the MMA warp
 * never signals that the first tile's scores are ready, so the softmax warps'
 * wait for them cannot complete.  The kernel's main-loop waits give up after
 * limit_ns of wall time; every role of the CTA then stops, the CTA waits for
 * its own tensor-core operations and TMA loads in flight (those waits keep
 * the normal 2 s limit), frees its tensor memory, records fault code 1 in the
 * device fault word and returns.  The outputs are incomplete.  Read the code
 * with ra_device_fault(); the CUDA context stays usable.
 *
 *   limit_ns  1000 <= limit_ns <= 1e10, else RA_ERR_SHAPE.
 */
ra_status ra_attn_abort_selftest(const void* q, const void* k, const void* v, void* o,
                                 float* lse, int64_t B, int64_t H, int64_t N, int64_t d, int P,
                                 int layout, int causal, float scale, int64_t limit_ns,
                                 void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RINGATTN_H_ */
