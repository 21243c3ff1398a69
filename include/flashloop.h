/*
 * flashloop.h -- C ABI of the FlashLoop lazy loop-r attention sublayer on
 * NVIDIA B200 (sm_100a).
 *
 * The operation is defined by "FlashLoop: Fast and Memory-Efficient Looped
 * Transformers via Lazy Updates" (Yang & Liu): token-sparse updates (§4.1,
 * App. D.1), loop-aware sparse attention (§4.2, App. D.2), cross-loop KV
 * residual quantisation (§4.3, App. D.3) and the GPU engine of App. G
 * (active-token execution, fused projections, packed low-bit KV streams read
 * directly by the attention kernels, fused decode selection).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates, never frees and never synchronises the host.  Every
 *    call is asynchronous on the given stream (a cudaStream_t passed as
 *    void*, NULL = legacy default stream).
 *  - bf16 tensors are passed as uint16_t bit patterns, fp16 scales likewise.
 *  - Device tensors start on a 32-byte boundary (cudaMalloc and PyTorch
 *    allocations start on 256 bytes); the attention calls return
 *    FLASHLOOP_ERR_INVALID_ARG for a query, numerator or output tensor that
 *    does not.
 *  - Layouts are row-major.  Hidden states X are [S, d_model]; linear weights
 *    are [out, in] (y = x W^T); head h owns columns [h*dh, (h+1)*dh).
 *  - A loop r (1-based) indexes per-loop arrays at position r-1.
 *  - Counts of active tokens stay on the device: each kernel reads them there
 *    and sizes its grid by the host-known upper bound (the capacity).
 *  - Return value: FLASHLOOP_OK or a negative flashloop_status.  Arguments
 *    are checked before any launch; a failed check launches nothing.
 *    Device-side checks (capacity overflow, an index outside [0, S)) set
 *    *err_word to a non-zero FLASHLOOP_DEVERR_* code; the caller reads it
 *    after synchronising.  Kernels never trap and never spin without bound.
 *  - Supported shapes: head_dim in {64, 128}, d_model = n_heads * head_dim,
 *    d_model % 128 == 0, bits in {8, 4, 2} (bits[0] must be 8),
 *    1 <= topk <= S.  Anything else returns FLASHLOOP_ERR_UNSUPPORTED.
 */
#ifndef FLASHLOOP_H
#define FLASHLOOP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FLASHLOOP_MAX_LOOPS 16
#define FLASHLOOP_GROUP 32

typedef enum flashloop_status {
  FLASHLOOP_OK = 0,
  FLASHLOOP_ERR_INVALID_ARG = -1, /* null pointer, bad loop index, sizes out of range */
  FLASHLOOP_ERR_UNSUPPORTED = -2, /* shape or bit width outside the supported set */
  FLASHLOOP_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed */
  FLASHLOOP_ERR_DEVICE = -4,      /* reported by flashloop_check_error_word */
  FLASHLOOP_ERR_ARCH = -5         /* the current device is not sm_100 */
} flashloop_status;

/* Codes a kernel may leave in *err_word. */
#define FLASHLOOP_DEVERR_CAPACITY 1 /* more active tokens than the loop's capacity */
#define FLASHLOOP_DEVERR_INDEX 2    /* a token or column index outside [0, S) */
#define FLASHLOOP_DEVERR_TIMEOUT 3  /* a bounded wait inside a pipelined kernel gave up */
#define FLASHLOOP_DEVERR_RANGE 4    /* an attention operand (q, or a rebuilt key or value, keys
                                       times log2(e)/sqrt(dh)) is NaN or beyond the largest fp16
                                       (65504): the tensor-core operands are fp16 */

/* Problem description.  Plain values, read on the host only. */
typedef struct flashloop_params {
  int32_t seq;      /* S: tokens of the sequence (prefill) or of the context (decode) */
  int32_t d_model;  /* = n_heads * head_dim */
  int32_t n_heads;
  int32_t head_dim; /* 64 or 128 */
  int32_t n_loops;  /* R, 1..FLASHLOOP_MAX_LOOPS */
  int32_t batch;    /* decode: number of sequences; prefill: 1 */
  float tau;        /* gate threshold on the relative L2 change */
  float rope_theta; /* RoPE base (1e4) */
  int32_t topk[FLASHLOOP_MAX_LOOPS];     /* column budget k_r per loop (loop 1 unused), non-increasing */
  int32_t bits[FLASHLOOP_MAX_LOOPS];     /* code width per loop: bits[0] = 8 (base); 8, 4 or 2 after */
  int32_t capacity[FLASHLOOP_MAX_LOOPS]; /* rows allocated for loop r's active list and residual stream */
  int32_t gate_topk; /* 0: the tau threshold gate; else top-k token retention keeping capacity[r-1] tokens */
  int32_t fixed_mass; /* 0: running (m, N, Z) update; else the fixed-mass form (see flashloop_sparse_attn_update) */
  int32_t attn_pairs; /* reserved, must be 0 (FLASHLOOP_ERR_UNSUPPORTED otherwise): the running update
                         takes one SM per work item */
  int32_t kv_scheme;  /* 0: INT8 base + INT4/INT2 symmetric residuals (flashloop_kv streams);
                         1: the pages' own setting (flashloop_paper_kv streams, see below; prefill only) */
} flashloop_params;

/* One quantised cache (K or V) of a sequence: the loop-1 base over every
 * token and, for loops r >= 2, a residual stream over the loop's active
 * tokens only, stored at the token's position in the active list.
 * Groups are 32 consecutive head_dim elements of one (token, head); a code is
 * two's complement; INT4 packs element 2t in the low nibble of byte t, INT2
 * element 4t+u in bits [2u, 2u+1] of byte t. */
typedef struct flashloop_kv {
  int8_t* base_codes;                          /* [S, H, dh] */
  uint16_t* base_scales;                       /* [S, H, dh/32] fp16 */
  uint8_t* res_codes[FLASHLOOP_MAX_LOOPS];     /* loop r: [capacity_r, H, dh*bits_r/8] */
  uint16_t* res_scales[FLASHLOOP_MAX_LOOPS];   /* loop r: [capacity_r, H, dh/32] fp16 */
} flashloop_kv;

/* One cache (K or V) in the pages' own setting [FlashLoop App. E "Quantization
 * setting"; the "Looping a Transformer Quadruples the Bill" page, §3]:
 * INT4 asymmetric codes in groups of 64 with an fp16 scale and an fp16 minimum
 * per group (value = code * scale + minimum, codes 0..15), the last
 * FLASHLOOP_PAPER_TAIL tokens kept in bf16 instead.
 *  - Body tokens t < body = S - tail (tail = min(FLASHLOOP_PAPER_TAIL, S)):
 *    loop 1 codes the values themselves, row t; loop r >= 2 codes the residual
 *    against the reconstruction of loop r-1 for the loop's active body tokens,
 *    row = the token's position in the loop's active list (its slot).
 *  - Keys are grouped per channel over 64 consecutive rows (row / 64 is the
 *    group; a last partial group takes its minimum and maximum over its rows);
 *    values per row over 64 consecutive channels.
 *  - Reconstruction of loop r: the loop-1 codes plus, in loop order, the
 *    residual of every loop 2..r where the token was active (float32); a tail
 *    token's value is the bf16 value stored at the latest loop <= r where it
 *    was active (every token is active at loop 1).
 * Codes are packed two per byte along head_dim (element 2i in the low nibble). */
#define FLASHLOOP_PAPER_GROUP 64
#define FLASHLOOP_PAPER_TAIL 64
typedef struct flashloop_paper_kv {
  uint8_t* codes[FLASHLOOP_MAX_LOOPS];   /* loop r: [rows_r, H, dh/2] (rows_1 = body, rows_r = capacity_r) */
  uint16_t* scale[FLASHLOOP_MAX_LOOPS];  /* fp16; keys [ceil(rows_r/64), H, dh], values [rows_r, H, dh/64] */
  uint16_t* minv[FLASHLOOP_MAX_LOOPS];   /* fp16, the layout of scale */
  uint16_t* tail[FLASHLOOP_MAX_LOOPS];   /* bf16 [tail, H, dh] at position t - body (rows of tokens
                                            inactive at loop r are not written) */
} flashloop_paper_kv;

/* Whole per-sequence state of the sublayer (all device memory, caller-owned;
 * a checkpoint is a copy of these buffers).
 * Slots: q, m, Z and N have three slots.  Loop 1 writes slot 0; loop r >= 2
 * reads slot sel(r-1) and writes slot sel(r), sel(r) = 1 + (r % 2), so the
 * loop-1 state is never overwritten and loops 2..R can be re-run. */
typedef struct flashloop_state {
  flashloop_kv k;
  flashloop_kv v;
  int32_t* active[FLASHLOOP_MAX_LOOPS]; /* loop r: ascending active tokens, first n_r valid, [capacity_r] */
  int32_t* slot[FLASHLOOP_MAX_LOOPS];   /* loop r: [S] position of the token in active[r-1], -1 if inactive */
  int32_t* n_active;                    /* [FLASHLOOP_MAX_LOOPS] device counts n_r */
  uint16_t* q[3];                       /* bf16 [S, H, dh] query slots */
  float* m[3];                          /* [H, S] running max */
  float* Z[3];                          /* [H, S] running denominator */
  float* N[3];                          /* [H, S, dh] running numerator */
  float* colmass[2];                    /* [H, S]: [0] dense loop-1 column mass, [1] latest sparse loop's */
  int32_t* cols[FLASHLOOP_MAX_LOOPS];   /* loop r: [H, k_r] ascending selected columns (loops that select) */
  uint16_t* O;                          /* bf16 [S, d_model] attention output (rows of inactive tokens kept) */
  uint16_t* Y;                          /* bf16 [S, d_model] output projection (rows of inactive tokens kept) */
  float* rope_cs;                       /* [S, dh/2] (cos, sin) pairs, see flashloop_rope_table */
  int32_t* err_word;                    /* device error word, 0 = no error */
  void* workspace;                      /* scratch, zero-filled once before first use */
  size_t workspace_bytes;               /* >= flashloop_workspace_bytes(params) */
  float* G[3];                          /* [H, S] selected-column factor g, one per m/Z/N slot
                                           (params.fixed_mass only; NULL otherwise) */
  /* params.kv_scheme == 1: the K and V streams in the pages' setting (k and v above are then
     unused).  The structs themselves are host memory, read on the host; the buffers they point
     to are device memory. */
  const flashloop_paper_kv* paper_k;
  const flashloop_paper_kv* paper_v;
} flashloop_state;

/* ---------------------------------------------------------------- sizing */

/* Scratch bytes the calls below need in state->workspace (host function; a
 * sizing helper, not an operation of the method). */
size_t flashloop_workspace_bytes(const flashloop_params* p);

/* Cache bytes of K and V for the given active counts n_r (n[0] = S):
 * base 2*S*H*(dh + 2*dh/32) plus, per loop r >= 2, 2*n_r*H*(dh*bits_r/8 + 2*dh/32).
 * Byte accounting of the cross-loop KV store ([FlashLoop §4.3, App. D.3]). */
size_t flashloop_cache_bytes(const flashloop_params* p, const int32_t* n_per_loop);

/* Fill the RoPE table: cs[2*(t*dh/2 + i)] = cos(t * theta^(-2i/dh)),
 * cs[2*(...)+1] = sin(...), for t < n_pos, computed in double precision and
 * rounded to float.  Rotate-half pairing (i, i + dh/2).  [FlashLoop App. E
 * quantises keys after RoPE; the pages fix no RoPE variant, and the
 * rotate-half form with theta = p->rope_theta and position = token index is
 * taken.]  cs: device, caller-owned, n_pos * dh floats. */
int flashloop_rope_table(const flashloop_params* p, int32_t n_pos, float* cs, void* stream);

/* ---------------------------------------------------------------- the path */

/* (a1, top-k retention) [FlashLoop §4.1 and App. D.1: a budget of tokens kept per loop]:
 * instead of the tau threshold, keep the `budget` candidates of largest
 * normalised change ||x_cur - x_prev||^2 / ||x_prev||^2 (float32 sums, IEEE
 * division; a zero previous row counts as +inf if it changed, 0 if not),
 * ties to the lower token.  Candidates are prev_active[0..*n_prev) (ascending),
 * or every token when prev_active is NULL.  Writes the kept tokens ascending
 * to active_out, every token's position to slot_out (-1 = not kept) and
 * min(budget, n_prev) to *n_active_out.  budget <= out_capacity,
 * prev_capacity <= 49152. */
int flashloop_gate_topk(const flashloop_params* p, const uint16_t* x_cur, const uint16_t* x_prev,
                        const int32_t* prev_active, const int32_t* n_prev, int32_t prev_capacity,
                        int32_t budget, int32_t* active_out, int32_t* slot_out, int32_t* n_active_out,
                        int32_t out_capacity, void* workspace, int32_t* err_word, void* stream);

/* (a1) Token change gate and stream compaction [FlashLoop §3.1, §4.1, App. D.1].
 * For the n_prev candidates prev_active[0..n_prev) (ascending), a token is
 * active iff sum_c (x_cur - x_prev)^2 >= tau^2 * sum_c x_prev^2 (float32
 * sums).  Writes the ascending active tokens to active_out, their positions
 * to slot_out (every one of the S entries is written, -1 = inactive) and
 * the count to *n_active_out.  prev_capacity bounds n_prev; out_capacity
 * bounds the output (overflow sets FLASHLOOP_DEVERR_CAPACITY and truncates). */
int flashloop_gate(const flashloop_params* p, const uint16_t* x_cur, const uint16_t* x_prev,
                   const int32_t* prev_active, const int32_t* n_prev, int32_t prev_capacity,
                   int32_t* active_out, int32_t* slot_out, int32_t* n_active_out, int32_t out_capacity,
                   void* workspace, int32_t* err_word, void* stream);

/* Variant of flashloop_gate for callers that cannot allocate device memory
 * (the paper has no counterpart: this is an interface for deployment).  Such
 * callers include a serving process that reserved all of HBM for its cache
 * pools at start-up and runs with a frozen budget, a host framework that owns
 * every device allocation, and latency-critical paths where cudaMalloc's
 * implicit device synchronisation is not acceptable.  The result is the same
 * as flashloop_gate's; there is no workspace argument.  Instead the
 * scratch (one byte per candidate and a ticket) lives in a file-scope device
 * array of the library: 64 KiB + 256 bytes that every GPU that loads the
 * library holds until the process exits.
 *  - Candidates (prev_capacity, or S when prev_active is NULL) above
 *    FLASHLOOP_NOALLOC_MAX_CANDIDATES return FLASHLOOP_ERR_UNSUPPORTED.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) and caches it with the current context; make
 *    that first call before any stream capture.  A call made in another
 *    context of that device (after cudaDeviceReset, or a new context) looks
 *    the address up again: the first call after such a change is again a
 *    set-up call and belongs before any capture.
 *  - Parameters, architecture and arguments are checked exactly as
 *    flashloop_gate checks them, with the same status codes.
 *  - Nothing is allocated or freed; each call zeroes the ticket with
 *    cudaMemsetAsync on `stream`, then launches the gate kernel.
 *  - Every call shares the one array, which keeps the previous call's
 *    contents: calls that overlap on the GPU (other streams, other host
 *    threads on the same device) race and must be serialised by the caller. */
#define FLASHLOOP_NOALLOC_MAX_CANDIDATES 65536
int flashloop_gate_noalloc(const flashloop_params* p, const uint16_t* x_cur, const uint16_t* x_prev,
                           const int32_t* prev_active, const int32_t* n_prev, int32_t prev_capacity,
                           int32_t* active_out, int32_t* slot_out, int32_t* n_active_out,
                           int32_t out_capacity, int32_t* err_word, void* stream);

/* (a2) Gathered Q/K/V projection with RoPE [FlashLoop §4.3 (post-RoPE keys),
 * App. E, App. G "fused projections"].  For a < *n_active, token t = active[a]:
 * [q|k|v] = x[t] W_qkv^T (W_qkv = [W_q; W_k; W_v], [3d, d]), float32
 * accumulation, RoPE at position t on q and k.  q is stored as bf16 at
 * q_out[t] ([S, H, dh]); k and v as float32 at k_out[a], v_out[a]
 * ([capacity, H, dh]).  active = NULL means the identity over S tokens. */
int flashloop_qkv_gathered(const flashloop_params* p, const uint16_t* x, const int32_t* active,
                           const int32_t* n_active, int32_t capacity, const uint16_t* w_qkv,
                           const float* rope_cs, uint16_t* q_out, float* k_out, float* v_out,
                           void* stream);

/* (a3) Cross-loop KV residual quantisation [FlashLoop §3.3, §4.3, App. D.3].
 * loop == 1: the INT8 base of k_new / v_new for every token (k_new[t]).
 * loop >= 2: for a < *n_active, token t = active[a]: rho = x_new[a] - Xhat^(r-1)_t
 * with Xhat^(r-1)_t = deq(base_t) + sum_{l=2}^{r-1} deq(res_l[slot_l[t]]) summed
 * in float32 in that order; s = fp16_rn(max|rho| / qmax) per group of 32,
 * code = clamp(rint(rho / s), -qmax, qmax) with IEEE float32 division
 * (s == 0 gives code 0), qmax = 2^(bits_r - 1) - 1; stored at res_r[a]. */
int flashloop_kv_quant_residual(const flashloop_params* p, int32_t loop, const float* k_new,
                                const float* v_new, const int32_t* active, const int32_t* n_active,
                                flashloop_state* st, void* stream);

/* (f2) The pages' own cache setting: quantisation of loop `loop`'s keys and
 * values into st->paper_k / st->paper_v (params.kv_scheme == 1; see
 * flashloop_paper_kv for the format).  k_new / v_new are float32 [rows, H, dh]
 * with row a the a-th token of active[0..*n_active) (loop 1: every token,
 * active may be NULL), keys after RoPE.  Body tokens are quantised (loop 1:
 * the values; loop r >= 2: the residual against the reconstruction of loop
 * r-1, with x - minimum and the division by the scale in IEEE float32 and
 * round-half-even, codes clamped to 0..15, a zero scale giving code 0); tail
 * tokens store bf16(x) in tail[loop-1].  The slot map of loop r (st->slot) must
 * hold the loop's active list.  [FlashLoop App. E; the "Quadruples the Bill"
 * page, §3.] */
int flashloop_paper_kv_quant(const flashloop_params* p, int32_t loop, const float* k_new, const float* v_new,
                             const int32_t* active, const int32_t* n_active, flashloop_state* st, void* stream);

/* (a2)+(a3) fused: the gathered projection of flashloop_qkv_gathered whose
 * epilogue quantises k and v of loop `loop` straight into the state's
 * streams (INT8 base at loop 1, the residual against Xhat^(loop-1) at loop
 * >= 2), with the same
 * arithmetic as flashloop_kv_quant_residual; q (RoPE'd, bf16) goes to
 * q_out[t].  [FlashLoop §4.3, §4.4: KV update fused with quantisation.]
 * The base row of token t is t; a residual row is slot[loop-1][t] (the
 * token's position in this loop's active list, written by the gate).
 * loop == 1 with active == NULL projects every token.  q_out may be NULL
 * (q is then not stored: a decode context needs only its K/V). */
int flashloop_qkv_quant(const flashloop_params* p, int32_t loop, const uint16_t* x, const int32_t* active,
                        const int32_t* n_active, const uint16_t* w_qkv, flashloop_state* st,
                        uint16_t* q_out, void* stream);

/* (a4) Column selection [FlashLoop §3.2, §4.2, App. D.2].  Per head h: the k
 * candidates of largest float32 mass[h, j] (ties to the lower index, -0 == +0),
 * written ascending to out[h*k ...].  candidates = NULL: all j in [0, S);
 * otherwise candidates[h*n_cand ...] ascending.  n (S or n_cand) <= 49152. */
int flashloop_topk_columns(const flashloop_params* p, const float* mass, const int32_t* candidates,
                           int32_t n_cand, int32_t k, int32_t* out, void* stream);

/* (a5) Selected-column reconstruction [FlashLoop App. G: attention reads the
 * packed anchor and residual streams, no full BF16 KV rebuild].  For loop
 * r >= 2 and each head h, rebuilds Khat^(r-1)_j, Khat^(r)_j, Vhat^(r-1)_j and
 * Vhat^(r)_j of the k selected columns j (cols of the latest selecting loop)
 * from the base and residual streams (float32 sums in loop order, rounded to
 * fp16) into state->workspace, where flashloop_sparse_attn_update reads them.
 * loop == 1 rebuilds Khat^(1), Vhat^(1) of every token. */
int flashloop_selcol_dequant(const flashloop_params* p, int32_t loop, flashloop_state* st,
                             void* stream);

/* (a6) Sparse attention update of loop r >= 2 [FlashLoop §3.2, §4.2,
 * App. D.2, App. G].  For each head h, active row i (tokens of active[r-1])
 * and selected column j <= i (cols of the latest selecting loop):
 *   s_old = q_i^(r-1) . Khat_j^(r-1) / sqrt(dh),  s_new = q_i^(r) . Khat_j^(r) / sqrt(dh),
 *   m' = max(m_i, max s_new), a = e^(m_i - m'),
 *   Z' = a Z_i - sum e^(s_old - m') + sum e^(s_new - m'),
 *   N' = a N_i - sum e^(s_old - m') Vhat_j^(r-1) + sum e^(s_new - m') Vhat_j^(r),
 *   O_i = N' / Z' (bf16).
 * Reads q slots sel(r-1), sel(r), the state slot sel(r-1) and the columns
 * flashloop_selcol_dequant rebuilt (call it first, same loop); writes the
 * state slot sel(r) and the rows of O.  With want_colmass != 0 also writes
 * colmass[1][h, j] = sum_i e^(s_new - m') / Z' for the selected j.
 * loop == 1 runs the dense loop-1 attention (every j <= i, no removal, the
 * state starts empty) and always writes colmass[0].
 *
 * With params.fixed_mass [FlashLoop §4.2: the selection's probabilities are
 * scaled to the mass the previous loop gave those columns]: the selected columns J of
 * row i keep the total probability they had after loop r-1 and share it in
 * proportion to e^(s_new); unselected columns keep theirs.  The state gains
 * g (G[slot], [H, S]), the weight of the selected columns relative to
 * e^(s - m) / Z (the dense loop writes g = 1):
 *   g' = g sum_J e^(s_old - m') / sum_J e^(s_new - m')   (g' = g when J is empty),
 *   Z' = a Z_i,
 *   N' = a N_i - g sum_J e^(s_old - m') Vhat_j^(r-1) + g' sum_J e^(s_new - m') Vhat_j^(r),
 * with m' any common frame (the call picks one that keeps the scaled
 * exponentials in fp16 range).  It runs as two launches, a statistics pass
 * and the update; colmass[1] then sums g' e^(s_new - m') / Z'. */
int flashloop_sparse_attn_update(const flashloop_params* p, int32_t loop, flashloop_state* st,
                                 int32_t want_colmass, void* stream);

/* (a7) Gathered output projection: for a < *n_active, t = active[a]:
 * y[t] = bf16(o[t] W_o^T) (float32 accumulation); other rows untouched.
 * [FlashLoop §4.1: active-token execution recomputes only the active rows;
 * the sublayer's output weight W_o completes the attention block.]
 * o, y: bf16 [S, d_model] (row = token); w_o: bf16 [d_model, d_model]. */
int flashloop_out_proj(const flashloop_params* p, const uint16_t* o, const int32_t* active,
                       const int32_t* n_active, int32_t capacity, const uint16_t* w_o, uint16_t* y,
                       void* stream);

/* One loop of the sublayer: a1..a7 at loop >= 2 (gate against x_prev), or the
 * dense setup at loop == 1 (x_prev unused): every token active, INT8 base,
 * dense causal attention on the reconstructed base, column mass, W_o.
 * With p->gate_topk the gate is flashloop_gate_topk with budget capacity[r-1]. 
 * [FlashLoop §4, App. D]. */
int flashloop_loop_step(const flashloop_params* p, int32_t loop, const uint16_t* x_cur,
                        const uint16_t* x_prev, const uint16_t* w_qkv, const uint16_t* w_o,
                        flashloop_state* st, void* stream);

/* The KV path of one loop, without attention: at loop 1 the INT8 base of
 * every token; at loop r >= 2 the gate of x_cur against x_prev over loop
 * r-1's active list (flashloop_gate) and the residual of the active tokens
 * (flashloop_qkv_quant with q_out = NULL).  Reads/writes st->k, st->v,
 * st->active, st->slot, st->n_active, st->workspace (the gate's part, see
 * flashloop_kv_workspace_bytes), st->rope_cs and st->err_word only.
 * [FlashLoop §4.3: the cross-loop KV store of the converged and active
 * tokens]; this is what a decode context keeps from its prefill. */
int flashloop_kv_step(const flashloop_params* p, int32_t loop, const uint16_t* x_cur, const uint16_t* x_prev,
                      const uint16_t* w_qkv, flashloop_state* st, void* stream);

/* Scratch bytes flashloop_kv_step needs in st->workspace (zero-filled once;
 * a sizing helper). */
size_t flashloop_kv_workspace_bytes(const flashloop_params* p);

/* ---------------------------------------------------------------- decode */

/* (a8) Decode state of B sequences, one new token each at position S =
 * p->seq (the context length), all device memory, caller-owned.
 * The token of sequence b has its own K/V streams: base row b, and for every
 * loop l >= 2 residual row b (the token is active at every loop).
 * q, m, Z and N use the slots of flashloop_state: loop 1 writes slot 0, loop
 * r >= 2 reads slot sel(r-1) and writes slot sel(r) = 1 + (r % 2).
 * m is kept in log2 units: m = max_j q.k_j * log2(e) / sqrt(dh), and
 * Z = sum_j 2^(s_j - m), so that e^(natural max) * Z is the softmax sum. */
typedef struct flashloop_decode_state {
  flashloop_kv k;            /* token streams: base [B, H, dh], residual of loop l [B, H, dh*bits_l/8] */
  flashloop_kv v;
  const float* rope_cs;      /* (cos, sin) pairs of position S: [dh/2][2] (row S of flashloop_rope_table) */
  uint16_t* q[3];            /* bf16 [B, H, dh] query slots */
  float* m[3];               /* [B, H] */
  float* Z[3];               /* [B, H] */
  float* N[3];               /* [B, H, dh] */
  float* probs;              /* [B, H, S+1] float32 loop-1 attention probabilities (flashloop_decode_select) */
  int32_t* cols;             /* [B, H, topk[1]] ascending selected columns in [0, S] (S = the token) */
  uint16_t* O;               /* bf16 [B, d_model] */
  uint16_t* Y;               /* bf16 [B, d_model] */
  int32_t* err_word;         /* device error word, 0 = no error */
  void* workspace;           /* scratch (need not be cleared); carries the selected columns' rebuilt
                                K/V from one loop to the next (see flashloop_decode_attn) */
  size_t workspace_bytes;    /* >= flashloop_decode_workspace_bytes(params) */
} flashloop_decode_state;

/* Scratch bytes of flashloop_decode_step / flashloop_decode_attn (host function;
 * a sizing helper).
 * p->batch = B in [1, 64]; additionally n_heads*head_dim must be a multiple of
 * 256 and n_heads*head_dim/32 a divisor of 256 that is a multiple of 8
 * (e.g. 16 x 128, 4 x 64); returns 0 for any other shape. */
size_t flashloop_decode_workspace_bytes(const flashloop_params* p);

/* (a8) Decode attention of loop `loop` [FlashLoop App. G: custom attention
 * kernels read the packed anchor and residual streams directly; fused sparse
 * decode selection].  ctx holds the B contexts' caches as one sequence of B*S
 * rows (token j of sequence b at row b*S + j; its loop-l residual at row
 * ctx->slot[l-1][b*S + j], -1 = none), written by the KV path of loops
 * 1..R (flashloop_gate, flashloop_qkv_quant with p->seq = B*S); only ctx->k,
 * ctx->v and ctx->slot are read.  Columns 0..S-1 are the context, column S is
 * the token itself (its streams in ds).
 * loop 1: dense attention of q (slot 0) over Khat^(1), Vhat^(1) of columns
 *   0..S (base codes dequantised in the loads): state slot 0, O; the scores
 *   stay in the workspace for flashloop_decode_select.
 * loop r >= 2: for the selected columns j,
 *   s_old = q^(r-1).Khat_j^(r-1)/sqrt(dh), s_new = q^(r).Khat_j^(r)/sqrt(dh),
 *   m' = max(m, max s_new), Z' = e^(m-m') Z - sum e^(s_old-m') + sum e^(s_new-m'),
 *   N' likewise with Vhat^(r-1), Vhat^(r); O = N'/Z' (bf16).  The selection
 *   is fixed after loop 1, so the rebuilt columns carry over: loop 2 rebuilds
 *   Khat^(1), Vhat^(1) from the INT8 base (float32) and adds the loop-2
 *   residual; loop r >= 3 starts from the Khat^(r-1), Vhat^(r-1) that loop r-1
 *   left in ds->workspace (fp16) and adds the loop-r residual (float32).  The
 *   loops of a step therefore run in order 1..R on one workspace.
 * Argument errors are returned before any launch; a column index outside
 * [0, S] sets FLASHLOOP_DEVERR_INDEX. */
int flashloop_decode_attn(const flashloop_params* p, int32_t loop, const flashloop_state* ctx,
                          flashloop_decode_state* ds, void* stream);

/* (a8) [FlashLoop App. G: the decode path] Projections of the decode token
 * at loop `loop`: q, k, v = x_tok W_qkv^T
 * (x_tok bf16 [B, d_model], float32 accumulation, RoPE at position S on q and
 * k; q -> ds->q slot of the loop); k and v quantised into the token streams
 * (INT8 base at loop 1, the residual against the reconstructed previous loop
 * after it, the arithmetic of flashloop_kv_quant_residual).  The token is
 * active at every loop (no gate). */
int flashloop_decode_qkv(const flashloop_params* p, int32_t loop, const uint16_t* x_tok, const uint16_t* w_qkv,
                         flashloop_decode_state* ds, void* stream);

/* (a8) Fused sparse decode selection [FlashLoop App. G]: cols = per
 * (sequence, head) the topk[1] columns of largest float32 loop-1 probability
 * (ties to the lower index, written ascending), and probs = those
 * probabilities, 2^(s_j - m) / Z from the loop-1 scores kept in the
 * workspace by flashloop_decode_attn (call it first).  Needs S + 1 <= 49152. */
int flashloop_decode_select(const flashloop_params* p, flashloop_decode_state* ds, void* stream);

/* (a8) [FlashLoop App. G: the decode path] Output projection of the decode
 * tokens: Y = bf16(O W_o^T), float32 accumulation. */
int flashloop_decode_out(const flashloop_params* p, const uint16_t* w_o, flashloop_decode_state* ds,
                         void* stream);

/* (a8) [FlashLoop App. G: the decode path, its sparse selection fused with
 * the dense loop-1 pass] One loop of the decode token, B sequences: flashloop_decode_qkv,
 * flashloop_decode_attn, flashloop_decode_select (loop 1, when R >= 2),
 * flashloop_decode_out. */
int flashloop_decode_step(const flashloop_params* p, int32_t loop, const uint16_t* x_tok,
                          const uint16_t* w_qkv, const uint16_t* w_o, const flashloop_state* ctx,
                          flashloop_decode_state* ds, void* stream);

/* Host helper: the loop whose selection loop r uses (2 <= r): the latest
 * loop l <= r with l == 2 or topk[l-1] < topk[l-2].  [FlashLoop §4.2: the
 * selection is re-ranked when the column budget shrinks, and kept otherwise.] */
int32_t flashloop_selection_loop(const flashloop_params* p, int32_t loop);

/* Copy *err_word to the host (synchronising the stream) and map it to a
 * status: FLASHLOOP_OK, or FLASHLOOP_ERR_DEVICE with the code in *code
 * (diagnostics; not an operation of the method). */
int flashloop_check_error_word(const int32_t* err_word, int32_t* code, void* stream);

/* Self-test of the bounded waits that every pipelined kernel of the library
 * uses (diagnostics; the paper has no counterpart).  One thread initialises a
 * shared-memory barrier that nothing ever completes and waits on it with the
 * library's spinning wait (kind 0, about 2^22 polls with back-off) or its
 * sleeping wait (kind 1, about 2^16 tries of up to 20 us); when the wait gives
 * up the kernel writes FLASHLOOP_DEVERR_TIMEOUT to *err_word and returns, so
 * the stream and the context stay usable.  Takes about a second on the GPU.
 * Returns FLASHLOOP_ERR_INVALID_ARG for another kind or a NULL err_word. */
int flashloop_selftest_bounded_wait(int32_t kind, int32_t* err_word, void* stream);

/* Static description of a status code (diagnostics). */
const char* flashloop_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FLASHLOOP_H */
