/*
 * tps.h -- C ABI of libtps.so: token-pruned attention for video diffusion
 * transformers on NVIDIA B200 (sm_100a).
 *
 * The path, per denoising step and layer:
 *   lipar_score   -> per-token relative-L1 change             (float32 [N])
 *   lipar_select  -> ascending active index list idx + count  (int32, device)
 *   lipar_group / lipar_schedule -> HSA step groups and per-step active list
 *   tps_gather_rows -> the active tokens' rows (input of the QKV projection)
 *   kv_sync       -> fresh K/V rows into the layer cache (+ noise-aware re-noise)
 *   kv_rerotate   -> cached keys of pruned tokens turned to their own RoPE position
 *   pruned_attn   -> active queries attend all N cached keys (optional key-block mask)
 *   scatter_out   -> active outputs written back over the cached outputs
 *
 * Sources (gist.science technical summaries):
 *   [LIPAR] "Training-free Latent Inter-Frame Pruning with Attention Recovery"
 *   [HSA]   "Resumen Tecnico: Asignacion de Pasos Heterogenea (HSA) para la
 *            Generacion Eficiente de Video"
 *   [SVOO]  "Training-Free Sparse Attention for Fast Video Generation via Offline
 *            Layer-Wise Sparsity Profiling and Online Bidirectional Co-Clustering"
 *   [TR]    "Timeripple: Accelerating vDiTs by Understanding the Spatio-Temporal
 *            Correlations in Latent Space"
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates device memory and keeps no pointer after the call returns.
 *     Exceptions are marked HOST.
 *   - bf16 tensors are IEEE bfloat16 bit patterns (tps_bf16), row-major.
 *     Token-major layouts: a K/V/Q/O row of token n is the H*d contiguous
 *     values of [N, H, d].
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream). Argument errors are detected on the host before any
 *     launch and leave all outputs untouched.
 *   - The active count lives in device memory (`count`, int32), so no host
 *     synchronisation is needed between stages; `cap` is the host-known upper
 *     bound of the count used to size grids. Rows j >= min(*count, cap) are
 *     ignored.
 *   - Index entries outside [0, N) are skipped by the kernels and recorded in
 *     a device status word (TPS_ERR_BOUNDS); tps_check() reports it.
 *   - Return value: one of the TPS_* status codes; tps_last_error() gives a
 *     message for the calling host thread.
 */
#ifndef TPS_H_
#define TPS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TPS_API __attribute__((visibility("default")))
#else
#define TPS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes --------------------------------------------------------- */
#define TPS_OK               0
#define TPS_ERR_INVALID_ARG  1  /* null pointer, bad mode, k > N, d not 64/128, ... */
#define TPS_ERR_SHAPE        2  /* sizes out of the supported range               */
#define TPS_ERR_ALIGN        3  /* a pointer is not 16-byte aligned               */
#define TPS_ERR_CUDA         4  /* a CUDA runtime/driver call failed (message)    */
#define TPS_ERR_TIMEOUT      5  /* a bounded device wait gave up (tps_check)      */
#define TPS_ERR_BOUNDS       6  /* an index outside [0, N) was skipped (tps_check)*/
#define TPS_ERR_WORKSPACE    7  /* workspace null or smaller than required        */

typedef uint16_t tps_bf16;   /* bfloat16 bit pattern                  */
typedef void*    tps_stream; /* cudaStream_t                          */

/* ---- step 1: token score ([LIPAR] 2.B; [HSA] 2.1) ---------------------------
 * Relative L1 change per token:  s = sum_c |cur_c - ref_c| / sum_c |ref_c|,
 * computed in fp32 from bf16. den = 0 gives 0 when num = 0, else +inf.
 *   x            [F, HW, C] bf16, the current latent tokens (N = F*HW).
 *   x_ref        NULL: inter-frame mode, token (f,p) against (f-1,p).
 *                non-NULL: inter-step mode, [F, HW, C] bf16, token n against
 *                x_ref[n] (e.g. the previous step's velocity prediction).
 *   x_prev_frame inter-frame only: [HW, C] bf16 reference for frame 0; NULL
 *                makes every frame-0 score +inf (always active).
 *   score        [F*HW] float32 output.
 * Requires C % 8 == 0, 8 <= C <= 4096, F*HW < 2^31, 16-byte aligned pointers. */
TPS_API int lipar_score(const tps_bf16* x, const tps_bf16* x_ref, const tps_bf16* x_prev_frame,
                int64_t F, int64_t HW, int64_t C, float* score, tps_stream stream);

/* ---- motion-robust inter-frame score ([LIPAR] 2.B: motion detection with
 * short- and long-term differences) ---------------------------------------------
 * s(f, p) = max(rel-L1 of x[f,p] vs x[f-1,p], rel-L1 of x[f,p] vs x[max(f-L,0),p]),
 * frame 0 = +inf; a token is pruned only when both changes are small. L >= 1
 * (L = 1 is lipar_score's inter-frame mode). x [F, HW, C] bf16, C in {64, 128};
 * score float32 [F*HW]. */
TPS_API int lipar_score_motion(const tps_bf16* x, int64_t F, int64_t HW, int64_t C, int L, float* score,
                               tps_stream stream);

/* ---- per-axis similarity check of Q or K tokens ([TR] Metodologia 2) ---------
 * Three independent checks per (token, head), along t, x and y. The neighbour on
 * an axis is the previous token on it: t -> (f-1, y, x), x -> (f, y, x-1),
 * y -> (f, y-1, x). Each check measures the root-mean-square difference over
 * a cyclic window of head channels,
 *   Delta_a = sqrt( sum_{c in W_a} (x[n,h,c] - x[nb_a(n),h,c])^2 / len_a ),
 *   W_a = { (start_a + j) mod d : 0 <= j < len_a },
 * and Delta_a = +inf when the token has no neighbour on the axis or len_a = 0.
 * fp32 arithmetic on bf16 inputs. A (token, head) is reusable iff Delta_a <
 * theta_a on ANY axis (logical OR).
 *   x        [F, Hs, Ws, H, d] bf16 (token-major [N, H, d], N = F*Hs*Ws,
 *            n = (f*Hs + y)*Ws + x), 16-byte aligned; d in {64, 128}.
 *   windows  HOST int32[6] = {start_t, len_t, start_x, len_x, start_y, len_y},
 *            0 <= start < d, 0 <= len <= d.
 *   theta    HOST float[3] = {theta_t, theta_x, theta_y}; not NaN. The check
 *            is strict, so theta <= 0 never passes.
 *   reuse    [N, H] uint8 output: bit a (0 = t, 1 = x, 2 = y) set iff
 *            Delta_a < theta_a.
 *   delta    [3, N, H] float32 output (Delta_t, Delta_x, Delta_y), or NULL.
 *   score    [N] float32 output, or NULL: the number of heads of token n
 *            whose reuse byte is 0 (an integer). lipar_select with threshold
 *            tau = 1 then keeps every token that needs any head recomputed.
 * The reading of the standard error as an RMS difference, the choice of
 * neighbours and the token score are stated readings: the summary leaves them
 * open. */
TPS_API int timeripple_score(const tps_bf16* x, int64_t F, int64_t Hs, int64_t Ws, int H, int d,
                             const int32_t* windows, const float* theta, uint8_t* reuse, float* delta,
                             float* score, tps_stream stream);

/* Threshold schedule ([TR] Metodologia 3): the thresholds rise linearly over a
 * window of steps and stay fixed outside it. Returns theta_lo for step <= i0,
 * theta_hi for step >= i1, and the linear interpolation in between (steps
 * counted from 1; the summary's window is i0 = 11, i1 = 21). Host-only, pure;
 * i1 <= i0 makes it a step at i0. */
TPS_API float timeripple_theta(int step, float theta_lo, float theta_hi, int i0, int i1);

/* ---- steps 2-3: active set and compaction ([LIPAR] 2.B; [HSA] 2.1) ---------
 * mode TPS_SELECT_THRESHOLD: active iff score >= tau (a token below tau is
 *   redundant and pruned). NaN is never active.
 * mode TPS_SELECT_TOPK: the k highest scores; equal scores go to the lower
 *   index; NaN ranks below -inf; -0 equals +0. 0 <= k <= N.
 * Output: idx[0 .. *count) ascending int32 token indices (idx must hold N
 *   entries for threshold mode, k for top-k), *count written on the device.
 * ws: device workspace, 16-byte aligned, of tps_workspace_size(TPS_OP_SELECT,
 *   N, 0) bytes; its contents need no initialisation. With that size a call of
 *   N <= 524,288 runs as one cooperative launch; a smaller workspace (down to
 *   the multi-launch minimum, else TPS_ERR_WORKSPACE) selects the multi-launch
 *   path, with identical results. Calls that share one workspace must be
 *   ordered on the GPU (same stream). */
#define TPS_SELECT_THRESHOLD 0
#define TPS_SELECT_TOPK      1
TPS_API int lipar_select(const float* score, int64_t N, int mode, float tau, int64_t k,
                 int32_t* idx, int32_t* count, void* ws, size_t ws_bytes, tps_stream stream);

/* Allocation-free variant of lipar_select (the pages have no counterpart; it
 * exists for callers that cannot allocate a workspace, e.g. a host running the
 * step inside a fixed device-memory plan, or a denoising loop that must not
 * call cudaMalloc because it synchronises the device). Same contract as
 * lipar_select, but the selection scratch is a file-scope device array inside
 * libtps.so sized for N <= 4,194,304 tokens (about 73 KB, held by every GPU
 * that loads the library until exit); larger N returns TPS_ERR_SHAPE. It
 * allocates nothing. The first call on each device looks up the array's
 * device address (with that device current), so make that first call before
 * any stream capture. Devices numbered 64 and above look the address up on
 * every call. The cached address does not survive cudaDeviceReset: do not
 * call this entry point after resetting a device. All calls on a device share
 * the one array: calls that overlap on the GPU (e.g. on two streams without
 * ordering) race; the scratch keeps the last call's contents and is
 * re-initialised by every call. */
TPS_API int lipar_select_static(const float* score, int64_t N, int mode, float tau, int64_t k,
                                int32_t* idx, int32_t* count, tps_stream stream);

/* ---- fused front end: steps 1-3 in one launch ([LIPAR] 2.B; [HSA] 2.1) ------
 * Exactly lipar_score(x, x_ref, x_prev_frame, F, HW, C) followed by
 *   mode TPS_FRONT_THRESHOLD / TPS_FRONT_TOPK: lipar_select (tau / k, idx,
 *     count as there), or
 *   mode TPS_FRONT_GROUP: lipar_group (K groups into group[N]).
 * score: NULL, or float32 [N] that also receives the scores.
 * For C in {64, 128} and N <= 524,288 this runs as ONE cooperative launch:
 * each block scores its own tokens (the same arithmetic as lipar_score, so
 * the scores are bit-identical) into shared memory and the selection or rank
 * split reads them there; otherwise the separate kernels run, with identical
 * results. ws: tps_workspace_size(TPS_OP_FRONT, N, K) bytes (K ignored except
 * for groups), 16-byte aligned; its contents need no initialisation. Calls
 * that share one workspace must be ordered on the GPU. */
#define TPS_FRONT_THRESHOLD 0
#define TPS_FRONT_TOPK      1
#define TPS_FRONT_GROUP     2
TPS_API int lipar_front(const tps_bf16* x, const tps_bf16* x_ref, const tps_bf16* x_prev_frame,
                        int64_t F, int64_t HW, int64_t C, int mode, float tau, int64_t k, int K,
                        float* score, int32_t* idx, int32_t* count, int8_t* group,
                        void* ws, size_t ws_bytes, tps_stream stream);

/* ---- HSA group assignment ([HSA] 2.1, dynamic token selection) -------------
 * Ranks tokens by score descending (ties to the lower index, NaN last) and
 * splits the ranks into K contiguous groups of N/K (the remainder joins the
 * last group). group[n] = 0 for the fastest-changing third (the reference
 * group G_1 with the full budget), K-1 for the slowest. 1 <= K <= 8, K <= N.
 * ws: tps_workspace_size(TPS_OP_GROUP, N, K) bytes. */
TPS_API int lipar_group(const float* score, int64_t N, int K, int8_t* group,
                void* ws, size_t ws_bytes, tps_stream stream);

/* ---- HSA per-step active set ([HSA] 2.1 schedule, 2.4 phase window) --------
 * Group k is active at global step `step` iff step mod (T / budgets[k]) == 0;
 * every group is active when step < m or step >= T - m.
 *   budgets  HOST int32[K], each a divisor of T (budgets[0] = T for G_1).
 *   group    [N] int8 from lipar_group (values outside [0, K) are never active).
 *   idx, count as for lipar_select (idx holds N entries).
 * ws: tps_workspace_size(TPS_OP_SCHEDULE, N, K) bytes. */
TPS_API int lipar_schedule(const int8_t* group, int64_t N, int K, const int32_t* budgets, int T,
                   int step, int m, int32_t* idx, int32_t* count,
                   void* ws, size_t ws_bytes, tps_stream stream);

/* ---- gather of active rows ([HSA] 2.2 (1): only active tokens enter the
 * QKV projection) --------------------------------------------------------------
 * dst[j] = src[idx[j]] for j < min(*count, cap); rows of row_bytes bytes
 * (row_bytes % 16 == 0); src has N rows, dst cap rows. src may also be pinned
 * host memory mapped into the device's address space (see
 * tps_pointer_is_device_accessible): only the active rows then cross PCIe. */
TPS_API int tps_gather_rows(void* dst, const void* src, const int32_t* idx, const int32_t* count,
                    int64_t cap, int64_t N, int64_t row_bytes, tps_stream stream);

/* ---- step 4: KV-cache synchronisation ([HSA] 2.2 (2); [LIPAR] 2.C) ---------
 * k_cache[idx[j]] = k_fresh[j] and v_cache[idx[j]] = v_fresh[j] for
 * j < min(*count, cap) (bit copies), caches [N, H, d], fresh [cap, H, d].
 * rn == NULL: nothing else; k_eff / v_eff are not touched (may be NULL).
 * rn != NULL (noise-aware duplication): additionally writes the attention
 *   inputs k_eff, v_eff [N, H, d]: active rows = the fresh rows; pruned rows
 *   n = bf16_rne(a * cache[n] + b * eps), eps ~ N(0,1) from Philox4x32-10
 *   (Salmon et al., SC'11) with counter (q mod 2^32, q div 2^32, step,
 *   tensor: 0 = K, 1 = V), key (seed mod 2^32, seed div 2^32), q = e div 4 for
 *   flat element e = (n*H + h)*d + c, word e mod 4 mapped to
 *   u = (floor(w/2^9) + 1/2) * 2^-23, Box-Muller over words (0,1) and (2,3).
 *   eps is computed in fp32 with the hardware log2, sine and cosine: it is
 *   within about 1e-5 of the exact Box-Muller value, before the bf16 rounding.
 *   The cache is not overwritten by noised rows. idx must be ascending.
 * d in {64, 128}; H*d <= 16384; N < 2^31. */
typedef struct tps_renoise {
  float    a;     /* weight of the clean cached row   */
  float    b;     /* weight of the fresh noise        */
  uint64_t seed;  /* Philox key                       */
  uint32_t step;  /* denoising step (counter word 2)  */
  uint32_t pad_;
} tps_renoise;

TPS_API int kv_sync(tps_bf16* k_cache, tps_bf16* v_cache, const tps_bf16* k_fresh,
            const tps_bf16* v_fresh, const int32_t* idx, const int32_t* count, int64_t cap,
            int64_t N, int H, int d, const tps_renoise* rn /* HOST, may be NULL */,
            tps_bf16* k_eff, tps_bf16* v_eff, tps_stream stream);

/* ---- attention recovery: keys reused across frames ([LIPAR] 2.C) -----------
 * "Training-free Latent Inter-Frame Pruning with Attention Recovery", Dutch
 * summary 2.C: the K/V of pruned tokens are approximated by the cached K/V of
 * the previous frame, taking the RoPE rotations into account; "Timeripple",
 * Metodologia 1: a head's rotary channels form temporal, x and y groups.
 * Writes k_eff [N, H, d] (bf16, may alias k_cache) from k_cache [N, H, d]:
 *   active rows n = idx[j], j < min(*count, cap): k_eff[n] = k_cache[n] (bit
 *     copy: after kv_sync these hold the fresh keys);
 *   every other row: k_cache[n] turned to its own position. Per head, the
 *     channels are the contiguous groups [t | x | y] of dims[0], dims[1],
 *     dims[2] channels (each even, summing to d); in group a the adjacent
 *     channels (o_a + 2j, o_a + 2j + 1) are rotated by
 *     phi = shift[a] * base^(-2j / dims[a]):
 *       (x, y) -> (x cos phi - y sin phi, x sin phi + y cos phi),
 *     computed in fp32 from an fp32 (cos, sin) table rounded from double
 *     precision, then rounded to bf16 (RNE).
 * A key cached at frame f-1 for the token at frame f takes shift = (1, 0, 0).
 * V needs no rotation (RoPE acts on Q and K only). idx must be ascending;
 * entries outside [0, N) or out of order raise TPS_ERR_BOUNDS at tps_check.
 * d in {64, 128}; H*d <= 16384; |shift[a]| <= 2^20; rope is a HOST pointer. */
typedef struct tps_rope {
  int32_t dims[3];   /* channels of the t, x and y rotary groups        */
  int32_t shift[3];  /* position offset: frames, columns, rows           */
  float   base;      /* frequency base (10000 in common video DiTs)      */
  int32_t pad_;
} tps_rope;

TPS_API int kv_rerotate(const tps_bf16* k_cache, const int32_t* idx, const int32_t* count, int64_t cap,
                        int64_t N, int H, int d, const tps_rope* rope, tps_bf16* k_eff, tps_stream stream);

/* ---- step 5: pruned attention ([HSA] 2.2 (3)-(4); [SVOO] part 2; [TR]) ------
 * For every active row j < min(*count, cap) and head h:
 *   o_act[j,h] = sum_n softmax_n(scale * q_act[j,h] . k[n,h]) v[n,h]
 * over all n < N, or, with a key-block mask, only over keys n whose block
 * n / block has blockmask[(idx[j] / block) * nb + n / block] != 0, where
 * nb = ceil(N / block): the mask row is the query's ORIGINAL token block.
 *   q_act  [cap, H, d] bf16; k, v [N, H, d] bf16; o_act [cap, H, d] bf16 (RNE).
 *   blockmask NULL (dense) or uint8 [nb, nb] (block must be 128, nb <= 4096).
 *   lse    NULL or float32 [cap, H]: natural-log sum of exp of the scaled
 *          logits. A row with no allowed key gets o = 0 and lse = -inf.
 * scale must be finite and > 0 (typically 1/sqrt(d)).
 * bf16 inputs, fp32 accumulation and softmax, tcgen05 tensor cores.
 * d in {64, 128}; 1 <= H <= 256; N < 2^31; pointers 16-byte aligned.
 * Dense launches whose last wave of 256-row query tiles x heads would be
 * mostly empty (e.g. a low keep ratio) split the key range S <= 4 ways over a
 * thread-block cluster whose CTAs merge their partial results over
 * distributed shared memory (no workspace): either the whole grid, or only
 * the query tiles left after the grid's full waves, in a second launch on the
 * same stream (tps_attn_plan reports which). Results agree with the unsplit
 * kernel within the attention tolerance.
 * With a mask, the active rows of each original query block (its run of the
 * ascending idx) are computed together against only the key blocks that query
 * block keeps: for d = 128 in units of at most 64 rows with the products
 * transposed (the 128 keys of a key tile as the MMA's M, the unit's rows as
 * N), for d = 64 in one 128-row tile per query block. */
TPS_API int pruned_attn(const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v,
                const int32_t* idx, const int32_t* count, int64_t cap, int64_t N, int H, int d,
                float scale, const uint8_t* blockmask, int block, tps_bf16* o_act, float* lse,
                tps_stream stream);

/* Same contract as pruned_attn, with a caller workspace that lets a launch
 * that would fill the GPU poorly (few query tiles x heads, e.g. a low keep
 * ratio) run as S <= 4 key-range splits in one grid plus an S-way
 * log-sum-exp merge (dense mode only). ws: device memory of
 * tps_attn_workspace_size(cap, N, H, d) bytes (0 when no split is chosen),
 * 16-byte aligned; with a smaller or NULL workspace the call runs unsplit.
 * Results agree with pruned_attn within the attention tolerance (the merge
 * rounds to bf16 once, from fp32 partials). */
TPS_API int pruned_attn_ws(const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v,
                           const int32_t* idx, const int32_t* count, int64_t cap, int64_t N, int H, int d,
                           float scale, const uint8_t* blockmask, int block, tps_bf16* o_act, float* lse,
                           void* ws, size_t ws_bytes, tps_stream stream);
TPS_API size_t tps_attn_workspace_size(int64_t cap, int64_t N, int H, int d);

/* The key-range split S (1..4) of the whole grid of a dense pruned_attn call
 * of this shape on the current device (1 = the grid is not split as a whole).
 * HOST query, no launch. */
TPS_API int tps_attn_split(int64_t cap, int64_t N, int H, int d);

/* The launch plan of a dense pruned_attn call of this shape on the current
 * device (HOST query, no launch): *split = whole-grid key split (1 = none);
 * *main_rows = rows [0, main_rows) of the unsplit launch (cap when there is no
 * tail launch); *tail_split = key split of the second launch that takes rows
 * [main_rows, cap) (1 = no second launch). Pointers are HOST, non-NULL.
 * Returns TPS_ERR_INVALID_ARG for a bad shape or a NULL pointer. */
TPS_API int tps_attn_plan(int64_t cap, int64_t N, int H, int d, int* split, int64_t* main_rows, int* tail_split);

/* Same contract as pruned_attn for dense attention with d = 128 (blockmask
 * must be NULL, else TPS_ERR_INVALID_ARG), computed on pairs of CTAs: one
 * tcgen05 MMA of M = 256 rows spans two SMs (cta_group::2), each SM holding
 * half of every K and V tile, and the probabilities P pass through shared
 * memory so that the next Q K^T overlaps the current softmax. Results agree
 * with pruned_attn within the attention tolerance; on B200 it runs at about
 * 0.6-0.7 of pruned_attn's throughput, and pruned_attn does not route to it. */
TPS_API int pruned_attn_pair(const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v,
                             const int32_t* idx, const int32_t* count, int64_t cap, int64_t N, int H, int d,
                             float scale, const uint8_t* blockmask, int block, tps_bf16* o_act, float* lse,
                             tps_stream stream);

/* Same contract as pruned_attn, computed with the legacy warp-level
 * mma.sync tensor-core path (kept as the baseline the tcgen05 kernel is
 * measured against). */
TPS_API int pruned_attn_mma(const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v,
                    const int32_t* idx, const int32_t* count, int64_t cap, int64_t N, int H,
                    int d, float scale, const uint8_t* blockmask, int block, tps_bf16* o_act,
                    float* lse, tps_stream stream);

/* ---- attention-recovery merge ([LIPAR] 2.C, log-sum-exp recovery) -------------
 * Exact merge of two attention results over DISJOINT key sets (e.g. two
 * pruned_attn calls over two key ranges): with w_i = exp(lse_i),
 *   o = (w1 o1 + w2 o2) / (w1 + w2),  lse = log(w1 + w2)   (fp32, bf16 output).
 * A part with lse = -inf contributes nothing; both -inf give o = 0, lse = -inf.
 * o1, o2, o bf16 [cap, H, d]; lse1, lse2, lse float32 [cap, H]; rows
 * j >= min(*count, cap) untouched. o may alias o1 or o2; lse (may be NULL)
 * must not alias lse1 / lse2. d in {64, 128}. */
TPS_API int attn_lse_merge(const tps_bf16* o1, const float* lse1, const tps_bf16* o2, const float* lse2,
                           const int32_t* count, int64_t cap, int H, int d, tps_bf16* o, float* lse,
                           tps_stream stream);

/* ---- step 6: restoration ([LIPAR] Dutch summary 2.D) -------------------------
 * o_full[idx[j]] = o_act[j] for j < min(*count, cap); every other row of
 * o_full [N, H, d] keeps its cached output bit for bit. o_full may also be
 * pinned, device-mapped host memory: only the active rows then cross PCIe. */
TPS_API int scatter_out(tps_bf16* o_full, const tps_bf16* o_act, const int32_t* idx,
                const int32_t* count, int64_t cap, int64_t N, int H, int d, tps_stream stream);

/* ---- HSA cached Euler update ([HSA] 2.3) -------------------------------------
 * Every token keeps the velocity of its most recent active step; each global
 * step advances ALL tokens by the same increment dsigma = sigma_{i+1} - sigma_i:
 *   v_cache[idx[j]] = v_fresh[j]        for j < min(*count, cap)  (bit copies)
 *   x[n] = fmaf(dsigma, v_cache[n], x[n]) for every n < N (one rounding)
 *   x        float32 [N, C], the sampler state (updated in place)
 *   v_cache  bf16 [N, C], velocity of each token's last active step (in place)
 *   v_fresh  bf16 [cap, C], velocities just predicted for the active tokens
 * idx must be ascending and unique; duplicates or entries outside [0, N) are
 * skipped and flagged (TPS_ERR_BOUNDS via tps_check). C % 8 == 0, C <= 4096. */
TPS_API int hsa_euler_update(float* x, tps_bf16* v_cache, const tps_bf16* v_fresh, const int32_t* idx,
                             const int32_t* count, int64_t cap, int64_t N, int64_t C, float dsigma,
                             tps_stream stream);

/* ---- support --------------------------------------------------------------- */
#define TPS_OP_SELECT   0
#define TPS_OP_GROUP    1
#define TPS_OP_SCHEDULE 2
#define TPS_OP_FRONT    3
/* Workspace bytes for lipar_select / lipar_group / lipar_schedule (0 on bad op). */
TPS_API size_t tps_workspace_size(int op, int64_t N, int K);

/* The smallest workspace those calls accept (0 on bad op): enough for the
 * multi-launch path only. Results are identical with either size. */
TPS_API size_t tps_workspace_min_size(int op, int64_t N, int K);

/* 1 if kernels of the current device may dereference p: device or managed
 * memory, or pinned host memory mapped into the device's address space at the
 * same address (the unified-addressing case); 0 otherwise (pageable host
 * memory, unknown pointers). Host-only query; it never faults. */
TPS_API int tps_pointer_is_device_accessible(const void* p);

/* Message of the last failing call on this host thread ("" if none). */
TPS_API const char* tps_last_error(void);

/* Synchronises `stream`, then reads and clears this device's status word:
 * TPS_OK, TPS_ERR_BOUNDS (an index was skipped) or TPS_ERR_TIMEOUT (a bounded
 * device wait gave up), or TPS_ERR_CUDA if the synchronisation failed. */
TPS_API int tps_check(tps_stream stream);

/* Debug export: the raw Philox4x32-10 words used by kv_sync's re-noise, for
 * counter blocks q0 .. q0+nq-1: out[4*i + w] = word w of block q0 + i. */
TPS_API int tps_philox_fill(uint32_t* out, uint64_t q0, int64_t nq, uint64_t seed, uint32_t step,
                    uint32_t tensor, tps_stream stream);

/* Self-test of the failure-detection path (no counterpart on the pages). One
 * CTA waits on a shared-memory barrier that nothing ever completes, through the
 * same bounded wait every library kernel uses, but with a limit of
 * limit_cycles SM clock cycles (clamped to [1000, 2e9]). The wait gives up,
 * the CTA records TPS_ERR_TIMEOUT in the status word and exits normally, so the
 * context stays usable; tps_check() then returns TPS_ERR_TIMEOUT once. */
TPS_API int tps_wait_probe(int64_t limit_cycles, tps_stream stream);

/* Test hook (host-side fault injection): the next n launches report
 * TPS_ERR_CUDA ("injected launch failure") instead of success. The kernels
 * still run; the hook exercises the error path of every entry point and of
 * its callers without faulting a GPU. n <= 0 clears it. */
TPS_API void tps_debug_inject_launch_failures(int n);

/* Library version string. */
TPS_API const char* tps_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TPS_H_ */
