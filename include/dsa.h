/*
 * dsa.h -- C ABI of the B200 (sm_100a) library for DeepSeek Sparse Attention
 * (DSA) layer stacks under IndexCache.
 *
 * Sources.  [IC] "读懂 IndexCache：从 DSA 的选词开销到跨层索引复用" (the
 * IndexCache explainer): §1.1 (F and S layers; the first layer must be F),
 * §1.2 and its Figure 2 loop (the index cache is set on F layers, read on S
 * layers; every layer attends with its own Q/K/V), §1.2's cost note (indexer
 * work O(N L^2) -> O(M L^2)).  [IDX] "注意力机制中的 Index：从位置下标到预算
 * 检索": §1 (visible set P_t = {s : 0 <= s < t}), §2 (sparse softmax over the
 * selected set S_t), §4 (lightning indexer score, TopK over s < t, MLA latent
 * rows shared by all query heads), §6.5 (top-k must be deterministic).
 *
 * Conventions shared by every entry point.
 *  - bf16 tensors are raw IEEE bfloat16 bit patterns (dsa_bf16); all tensors
 *    are dense, row-major, in DEVICE memory unless stated otherwise, and must
 *    be 16-byte aligned.
 *  - Query row i of a sequence sits at absolute position t = start_pos + i and
 *    may see key positions s < t (t <= Lk is required).  Prefill: start_pos =
 *    0, Lq = Lk.  Decode: Lq = 1, start_pos = Lk.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream), allocates nothing and never synchronises.  The caller
 *    owns every buffer, including the workspace and the index cache.
 *  - Argument errors are reported before anything is enqueued.  A kernel whose
 *    bounded internal wait expires records it in a device error word and
 *    returns early; dsa_check_device_errors() reports it as DSA_ERR_TIMEOUT.
 *  - Results are deterministic: the same inputs give bit-identical indices
 *    and outputs on every run ([IDX] §6.5).
 *  - The library is not re-entrant across host threads for dsa_last_error().
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t dsa_bf16;

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misalignment */
  DSA_ERR_BAD_PATTERN = 2, /* pattern empty, not 'F'/'S', or pattern[0] != 'F' */
  DSA_ERR_UNSUPPORTED = 3, /* shape outside what the kernels implement */
  DSA_ERR_WORKSPACE = 4,   /* ws_bytes below the *_workspace() requirement */
  DSA_ERR_CUDA = 5,        /* a CUDA runtime/driver call or launch failed */
  DSA_ERR_TIMEOUT = 6      /* a kernel's bounded wait expired (device word) */
} dsa_status;

/* Human-readable description of the most recent non-OK status. */
const char *dsa_last_error(void);

/* ---------------------------------------------------------------------------
 * Lightning indexer + top-k (F layers).  [IDX] §4: for each query row t,
 *   I[t,s] = sum_{j<H_I} w[t,j] * ReLU(q_idx[t,j,:] . k_idx[s,:]),  s < t,
 *   S_t = TopK_k { I[t,s] }.
 * Output row idx[b,i,:] lists the selected positions in ascending order,
 * followed by -1 padding when fewer than k positions are visible; equal
 * scores prefer the lower position (-0.0 equals +0.0).  Scores are formed in
 * fp32 from bf16 products (exact for integer-valued inputs and power-of-two
 * weights).  The L x L score matrix is never written.  Scale factors such as
 * d_I^-1/2 or H_I^-1/2 are folded into w by the caller (ReLU(c x) = c ReLU(x)
 * for c > 0).
 *   q_idx [B, Lq, H_I, d_I] bf16;  k_idx [B, Lk, d_I] bf16;  w [B, Lq, H_I] f32
 *   idx   [B, Lq, k] int32 (written)
 * Supported: H_I in {4, 8, 16, 32, 64}; d_I in {32, 64, 128}; 1 <= k <= 2048;
 * B >= 1; Lq >= 1; start_pos >= 0; start_pos + Lq - 1 <= Lk.
 * When every row sees at most k positions (start_pos + Lq - 1 <= k), TopK
 * keeps all of them: the rows are written directly and q_idx, k_idx and w
 * are not read (the short-prefill case, where the selection equals the
 * causal mask of dense attention).
 * Workspace: dsa_indexer_topk_workspace() bytes, contents undefined on entry. */
size_t dsa_indexer_topk_workspace(int B, int Lq, int Lk, int start_pos, int H_I,
                                  int d_I, int k);
dsa_status dsa_indexer_topk(const dsa_bf16 *q_idx, const dsa_bf16 *k_idx,
                            const float *w, int B, int Lq, int Lk, int start_pos,
                            int H_I, int d_I, int k, int32_t *idx, void *ws,
                            size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * Sparse core attention.  [IDX] §2: for each query row t and head h,
 *   e_r   = scale * q[t,h,:] . K[S_t[r], 0:D_qk]      (valid r: S_t[r] >= 0)
 *   out[t,h,:] = sum_r softmax_r(e) * V[S_t[r], 0:D_v]
 *   lse[t,h]   = log sum_r exp(e_r)  (natural log; -inf for an empty set)
 * An empty set gives out = 0.  MLA ([IDX] §4): pass k = v = the latent cache
 * with row stride 576, D_qk = 576, D_v = 512 (V is the first 512 columns);
 * every query head reads the same latent row.  Index rows come from
 * dsa_indexer_topk (any order is accepted; -1 entries are skipped, and so
 * are entries outside [0, Lk), which would name rows of another sequence or
 * none; causal use needs 0 <= S_t[r] < t).
 * Numerics: each score is an fp32 sum of exact bf16 products (the MLA kernel
 * splits the 576 columns over two CTAs and adds their fp32 partial sums, so
 * no intermediate is narrowed and no input range is imposed beyond finite
 * fp32 scores); the softmax runs in fp32, the weights are rounded to bf16 for
 * the P.V product (fp32 accumulation), the output to bf16.
 *   q   [B, Lq, n_h, D_qk] bf16
 *   kbuf rows: kbuf + (b*Lk + s)*k_row_stride, D_qk bf16 each
 *   vbuf rows: vbuf + (b*Lk + s)*v_row_stride, D_v bf16 each
 *   idx [B, Lq, k] int32;  out [B, Lq, n_h, D_v] bf16 (written)
 *   lse [B, Lq, n_h] f32 (written; may be NULL)
 * Supported: (n_h, D_qk, D_v) = (128, 576, 512) with kbuf == vbuf, or
 * n_h <= 128 with D_qk, D_v <= 128; k >= 1; row strides multiples of 8.
 * Rows are read up to min(t, k) entries: valid entries first, -1 after.
 * Workspace: dsa_sparse_attn_workspace() bytes. */
size_t dsa_sparse_attn_workspace(int B, int Lq, int n_h, int D_v, int k);
dsa_status dsa_sparse_attn(const dsa_bf16 *q, const dsa_bf16 *kbuf,
                           int64_t k_row_stride, const dsa_bf16 *vbuf,
                           int64_t v_row_stride, const int32_t *idx, int B,
                           int Lq, int Lk, int start_pos, int n_h, int D_qk,
                           int D_v, int k, float scale, dsa_bf16 *out,
                           float *lse, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * The IndexCache layer loop.  [IC] §1.1-§1.2, Figure 2:
 *   for each layer l: if pattern[l] == 'F': idx_cache = TopK(indexer_l)
 *                     out_l = sparse_attention_l(q_l, K_l, V_l, idx_cache)
 * S layers launch no indexer work and read idx_cache in place: no copy and
 * no memory beyond the single caller-owned idx_cache [B, Lq, k] int32.  On
 * return (stream order) idx_cache holds the last F layer's indices.
 * Projections, normalisation and the FFN between layers are outside this
 * library; each layer's tensors are given directly in `layers`.
 * pattern: n_layers characters 'F' or 'S' (no terminator needed), first 'F'.
 * For S layers q_idx/k_idx/w are ignored and may be NULL.
 * Workspace: indexcache_forward_workspace() bytes (shared by all layers). */
typedef struct {
  int B, Lq, Lk, start_pos; /* batch and positions, as above */
  int H_I, d_I, k;          /* indexer heads, head dim, top-k budget */
  int n_h, D_qk, D_v;       /* main attention heads and dims */
  float scale;              /* main-attention logit scale */
  int64_t k_row_stride, v_row_stride; /* element strides of K / V rows */
} dsa_dims;

typedef struct {
  const dsa_bf16 *q_idx; /* [B, Lq, H_I, d_I]   F layers only */
  const dsa_bf16 *k_idx; /* [B, Lk, d_I]        F layers only */
  const float *w;        /* [B, Lq, H_I]        F layers only */
  const dsa_bf16 *q;     /* [B, Lq, n_h, D_qk] */
  const dsa_bf16 *kbuf;  /* K rows (see dsa_sparse_attn) */
  const dsa_bf16 *vbuf;  /* V rows; == kbuf for MLA */
  dsa_bf16 *out;         /* [B, Lq, n_h, D_v] */
  float *lse;            /* [B, Lq, n_h] or NULL */
} dsa_layer_io;

size_t indexcache_forward_workspace(const dsa_dims *dims);
dsa_status indexcache_forward(const char *pattern, int n_layers,
                              const dsa_layer_io *layers, const dsa_dims *dims,
                              int32_t *idx_cache, void *ws, size_t ws_bytes,
                              void *stream);

/* ---------------------------------------------------------------------------
 * Variable-length batches.  [IDX] §4.3 (the cost account of DSA, with its
 * note that prefill and decode requests are served differently): a serving
 * batch mixes sequences of different lengths and positions.  The pages
 * describe one sequence at a time; a batch is the same computation applied
 * to each sequence independently.  Rows of all sequences are packed:
 *   query-side tensors (q_idx, w, q, out, lse, idx) hold the rows of
 *   sequence b at rows cu_q[b] .. cu_q[b+1]-1, in order; row i of sequence b
 *   sits at absolute position t = start_pos[b] + i and sees s < t;
 *   key-side tensors (k_idx, the K/V or latent rows) hold sequence b's
 *   cached positions s = 0 .. at rows cu_k[b] + s, s < cu_k[b+1] - cu_k[b].
 * The three arrays are DEVICE int32 arrays the caller owns; the host values
 * total_q = cu_q[B], total_k = cu_k[B] and the bounds max_Lq >= every
 * cu_q[b+1]-cu_q[b] and max_Lk >= every cu_k[b+1]-cu_k[b] size the launch.
 * Contract, checked on the device by dsa_check_varlen (the host cannot read
 * the arrays without synchronising): cu_q and cu_k start at 0, never
 * decrease and end at total_q / total_k; start_pos[b] >= 0; start_pos[b] +
 * (cu_q[b+1]-cu_q[b]) - 1 <= cu_k[b+1]-cu_k[b]; the per-sequence lengths
 * respect the bounds.  A batch breaking it gets unspecified rows but no
 * access outside the tensors.  Sequences with no query rows are allowed.
 * When every sequence has exactly one query row (max_Lq = 1, total_q = B:
 * decode), the indexer takes the streaming decode kernels. */
typedef struct {
  int B;                    /* sequences */
  const int32_t *cu_q;      /* device [B + 1] query-row offsets */
  const int32_t *cu_k;      /* device [B + 1] cached-row offsets */
  const int32_t *start_pos; /* device [B] position of each sequence's first row */
  int total_q, total_k;     /* cu_q[B], cu_k[B] */
  int max_Lq, max_Lk;       /* bounds of the per-sequence lengths */
} dsa_varlen;

/* dsa_indexer_topk over a variable-length batch: q_idx [total_q, H_I, d_I],
 * k_idx [total_k, d_I], w [total_q, H_I], idx [total_q, k] (written), with
 * the semantics, limits and row form of dsa_indexer_topk per sequence. */
size_t dsa_indexer_topk_varlen_workspace(const dsa_varlen *vl, int H_I, int d_I, int k);
dsa_status dsa_indexer_topk_varlen(const dsa_bf16 *q_idx, const dsa_bf16 *k_idx,
                                   const float *w, const dsa_varlen *vl, int H_I,
                                   int d_I, int k, int32_t *idx, void *ws,
                                   size_t ws_bytes, void *stream);

/* dsa_sparse_attn over a variable-length batch: q [total_q, n_h, D_qk],
 * K/V rows kbuf + r * k_row_stride for r < total_k (sequence b's position s
 * at r = cu_k[b] + s), idx [total_q, k], out [total_q, n_h, D_v], lse
 * [total_q, n_h] (may be NULL).  Index entries outside [0, the sequence's
 * cache length) are skipped. */
size_t dsa_sparse_attn_varlen_workspace(const dsa_varlen *vl, int n_h, int D_v, int k);
dsa_status dsa_sparse_attn_varlen(const dsa_bf16 *q, const dsa_bf16 *kbuf,
                                  int64_t k_row_stride, const dsa_bf16 *vbuf,
                                  int64_t v_row_stride, const int32_t *idx,
                                  const dsa_varlen *vl, int n_h, int D_qk, int D_v,
                                  int k, float scale, dsa_bf16 *out, float *lse,
                                  void *ws, size_t ws_bytes, void *stream);

/* indexcache_forward over a variable-length batch: the layer loop above with
 * packed per-layer tensors.  dims supplies H_I, d_I, k, n_h, D_qk, D_v, scale
 * and the row strides; its B, Lq, Lk and start_pos are ignored (vl gives
 * them).  idx_cache is [total_q, k]. */
size_t indexcache_forward_varlen_workspace(const dsa_dims *dims, const dsa_varlen *vl);
dsa_status indexcache_forward_varlen(const char *pattern, int n_layers,
                                     const dsa_layer_io *layers, const dsa_dims *dims,
                                     const dsa_varlen *vl, int32_t *idx_cache, void *ws,
                                     size_t ws_bytes, void *stream);

/* Checks the contract of a variable-length batch on the device and writes
 * the number of sequences that break it to *bad_seqs (one device int,
 * overwritten; read it after the stream completes).  Allocates nothing. */
dsa_status dsa_check_varlen(const dsa_varlen *vl, int *bad_seqs, void *stream);

/* ---------------------------------------------------------------------------
 * Low-precision selector.  [IDX] §5.4: the indexer's QK product on FP4 (or
 * FP8) operands and the index score quantised from FP32 to BF16 before the
 * top-k, trading exactness of the selection for speed.  The pages name the
 * formats only; the element and scale rules here are those of the OCP
 * Microscaling (MX) v1.0 format that block-scaled tensor-core products use:
 * along d_I, every 32 consecutive elements of a row share the power-of-two
 * scale X = 2^(floor(log2 amax) - emax) (emax = 8 for E4M3, 2 for E2M1),
 * held as an 8-bit exponent; each element becomes the format value nearest
 * to x / X (ties to even, saturating).  Then, per query row t,
 *   I[t,s] = bf16( sum_j w[t,j] * ReLU(q~[t,j,:] . k~[s,:]) )
 * over s < t (q~, k~ the dequantised values; the head dots are fp32 sums of
 * exact products), and S_t = TopK_k with the tie rule and row form of
 * dsa_indexer_topk.  Inputs, output and row conventions are those of
 * dsa_indexer_topk; the call quantises q_idx and k_idx into the workspace.
 * Supported: H_I = 64, d_I = 128, k <= 2048, fmt DSA_FMT_E4M3 or
 * DSA_FMT_E2M1.  Integer inputs in [-4, 4] quantise without loss. */
#define DSA_FMT_E4M3 0
#define DSA_FMT_E2M1 1
size_t dsa_indexer_topk_lowprec_workspace(int B, int Lq, int Lk, int start_pos, int H_I,
                                          int d_I, int k, int fmt);
dsa_status dsa_indexer_topk_lowprec(const dsa_bf16 *q_idx, const dsa_bf16 *k_idx,
                                    const float *w, int B, int Lq, int Lk, int start_pos,
                                    int H_I, int d_I, int k, int fmt, int32_t *idx, void *ws,
                                    size_t ws_bytes, void *stream);

/* MX quantisation of bf16 rows (the rule above): x [rows, cols] bf16 ->
 * codes [rows, cols] bytes and scales [rows, cols / 32] (the block exponent
 * E as E + 127).  E4M3: one code per byte.  E2M1: element 16 g + j of a row
 * sits in byte 16 g + j / 2 (the low nibble for even j), and bytes
 * 16 g + 8 .. 16 g + 15 are zero (the layout block-scaled tensor-core
 * products read 4-bit operands in).  Supported: cols = 128. */
dsa_status dsa_mx_quantize(const dsa_bf16 *x, int64_t rows, int cols, int fmt,
                           uint8_t *codes, uint8_t *scales, void *stream);

/* ---------------------------------------------------------------------------
 * Allocation-free variant of dsa_indexer_topk.  The pages describe no such
 * entry point; it exists for callers that cannot provide device memory on
 * demand -- an engine whose allocator already owns all of HBM, a C program
 * without an allocator, or a path that must avoid cudaMalloc/cudaFree because
 * they can synchronise the device.  Same inputs, output and semantics as
 * dsa_indexer_topk, but the scratch lives in a fixed device array inside the
 * library of DSA_NOALLOC_SCRATCH_BYTES (72 MiB, held on every GPU that loads
 * the library until the process exits); that covers k <= 2048 for prefill
 * shapes on up to 160 SMs and decode rows (Lq = 1) up to B * Lk of about
 * 18 million cached positions.  Shapes needing more return
 * DSA_ERR_WORKSPACE before anything is enqueued.  The first call on a device
 * looks up the array's device address (make it before any stream capture).
 * All calls share the array: calls whose kernels overlap on the GPU (other
 * streams, other host threads) race on it and must be serialised.  The
 * library allocates nothing on this path. */
#define DSA_NOALLOC_SCRATCH_BYTES (72u * 1024u * 1024u)
dsa_status dsa_indexer_topk_noalloc(const dsa_bf16 *q_idx, const dsa_bf16 *k_idx,
                                    const float *w, int B, int Lq, int Lk,
                                    int start_pos, int H_I, int d_I, int k,
                                    int32_t *idx, void *stream);

/* Number of dsa_indexer_topk launches issued by this process so far (host
 * counter; lets callers check that S layers run no indexer work). */
long long dsa_indexer_launch_count(void);

/* Validation of index rows (a debugging aid; the pages describe none):
 * counts the rows of idx [B, Lq, k] (device) that are not in the canonical
 * form dsa_indexer_topk writes -- for row i at t = start_pos + i, the first
 * min(t, k) entries strictly ascending in [0, t) ([IDX] §4: S_t is a subset
 * of {s : 0 <= s < t}), then -1 -- and writes the count to *bad_rows (one
 * device int, overwritten; read it after the stream completes).  Reads idx
 * only; allocates nothing. */
dsa_status dsa_check_indices(const int32_t *idx, int B, int Lq, int start_pos,
                             int k, int *bad_rows, void *stream);

/* ---------------------------------------------------------------------------
 * CSA-style selection over compressed blocks ([IDX] §5.2).  Every m tokens'
 * KV are compressed into one entry (the gated compression needs trained
 * weights and is not computed here: the compressed indexer keys and latent
 * entries are inputs).  Query row i at t = start_pos + i sees the compressed
 * blocks s < floor(t/m):
 *   I[t,s] = sum_j w[t,j] * ReLU(q_idx[t,j,:] . k_cmp[s,:]),
 *   S_t^CSA = TopK_k { I[t,s] : s < floor(t/m) },
 * with the tie rule and row form of dsa_indexer_topk, and the main attention
 * reads the selected compressed entries as shared K and V.
 *   q_idx [B, Lq, H_I, d_I] bf16; k_cmp [B, N_cmp, d_I] bf16; w [B, Lq, H_I]
 *   f32; idx [B, Lq, k] int32 (written).
 * Requires floor((start_pos + Lq - 1) / m) <= N_cmp, m >= 1, and the
 * dsa_indexer_topk limits on H_I, d_I, k.  Several query rows (Lq > 1) with
 * m > 1 need start_pos to be a multiple of m (chunked prefill on block
 * boundaries), else DSA_ERR_UNSUPPORTED.  The rows are regrouped by t mod m
 * into m sequences of one fused indexer launch, so the workspace holds a
 * phase-major copy of q_idx, w and the keys besides the indexer's own. */
size_t dsa_csa_indexer_topk_workspace(int B, int Lq, int N_cmp, int start_pos,
                                      int m, int H_I, int d_I, int k);
dsa_status dsa_csa_indexer_topk(const dsa_bf16 *q_idx, const dsa_bf16 *k_cmp,
                                const float *w, int B, int Lq, int N_cmp,
                                int start_pos, int m, int H_I, int d_I, int k,
                                int32_t *idx, void *ws, size_t ws_bytes,
                                void *stream);

/* Attention over the selected compressed entries ([IDX] §5.2, CoreAttn with
 * keys and values from the same entries): dsa_sparse_attn over the rows
 * c_cmp + (b*N_cmp + s)*row_stride, with the CSA visibility check above.
 * Valid index entries must satisfy 0 <= s < floor(t/m).  Workspace:
 * dsa_sparse_attn_workspace(B, Lq, n_h, D_v, k). */
dsa_status dsa_csa_sparse_attn(const dsa_bf16 *q, const dsa_bf16 *c_cmp,
                               int64_t row_stride, const int32_t *idx, int B,
                               int Lq, int N_cmp, int start_pos, int m, int n_h,
                               int D_qk, int D_v, int k, float scale,
                               dsa_bf16 *out, float *lse, void *ws,
                               size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * Selection quality ([IDX] §8, how index quality is evaluated).  Tools for short
 * contexts; they are not on the layer loop's path and run on CUDA cores.
 *
 * dsa_dense_weights: dense causal attention statistics of each query row
 * (row i at t = start_pos + i sees s < t; q, kbuf, k_row_stride as in
 * dsa_sparse_attn):
 *   lse_dense [B, Lq, n_h] f32 (written): log sum_{s<t} exp(scale q[t,h].K[s])
 *     (natural log; -inf for t = 0);
 *   mean_w [B, Lq, Lk] f32 (written for s < t only; may be NULL): the dense
 *     weights alpha^dense_{t,s} of §8.1 averaged over heads,
 *     (1/n_h) sum_h exp(scale q[t,h].K[s] - lse_dense[t,h]).
 * Supported: n_h <= 128, D_qk <= 576 and a multiple of 8, k_row_stride a
 * multiple of 8.  Work is O(sum_t t * n_h * D_qk) per pass, two passes. */
dsa_status dsa_dense_weights(const dsa_bf16 *q, const dsa_bf16 *kbuf,
                             int64_t k_row_stride, int B, int Lq, int Lk,
                             int start_pos, int n_h, int D_qk, float scale,
                             float *lse_dense, float *mean_w, void *stream);

/* dsa_topk_rows: TopK_k over dense score rows, the oracle selection of §8.2
 * (S^oracle = TopK_k of alpha^dense over s < t) when given mean_w.  Row
 * (b, i) is scores + (b*Lq + i)*row_stride and holds t = start_pos + i
 * finite scores; requires start_pos + Lq - 1 <= row_stride.  Output
 * idx [B, Lq, k] int32 in the row form of dsa_indexer_topk: ties go to the
 * lower position, positions ascending, then -1. */
dsa_status dsa_topk_rows(const float *scores, int64_t row_stride, int B, int Lq,
                         int start_pos, int k, int32_t *idx, void *stream);

/* dsa_index_overlap: inter[r] = |A_r & B_r| for `rows` pairs of index rows
 * of length k in the row form above (ascending, then -1; rows that are not
 * give an unspecified count but no out-of-range read).  inter / k is the
 * adjacent-layer overlap of §8.4 for A = S^(l), B = S^(l+1); inter /
 * |S^oracle| is Recall@k of §8.2 for A = S^oracle, B = S^model. */
dsa_status dsa_index_overlap(const int32_t *a, const int32_t *b, int64_t rows,
                             int k, int32_t *inter, void *stream);

/* dsa_captured_mass: CapturedMass@k of §8.1 per (row, head):
 * mass[e] = exp(lse_sel[e] - lse_dense[e]), which equals the dense weight
 * sum over the selected set when lse_sel comes from dsa_sparse_attn on that
 * set and lse_dense from dsa_dense_weights with the same q, K and scale.  A
 * row that sees nothing (lse_dense = -inf) gets mass 1.  MissedMass@k is
 * 1 - mass.  n elements, all f32 device arrays. */
dsa_status dsa_captured_mass(const float *lse_sel, const float *lse_dense,
                             int64_t n, float *mass, void *stream);

/* Self-test of failure detection (no counterpart in the pages): launches one
 * CTA that waits on a barrier nothing ever completes, gives up after
 * `limit_cycles` SM clock cycles (1 .. 2e9) and records the expiry in the
 * device error word exactly as the library's kernels do when one of their
 * bounded waits runs out.  The next dsa_check_device_errors() on `stream`
 * then returns DSA_ERR_TIMEOUT, and the context stays usable.  Nothing traps
 * or faults. */
dsa_status dsa_selftest_wait_timeout(long long limit_cycles, void *stream);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns DSA_ERR_TIMEOUT if any kernel's bounded wait expired since the last
 * call, DSA_ERR_CUDA on a CUDA error, DSA_OK otherwise. */
dsa_status dsa_check_device_errors(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
