/*
 * sa.h - C ABI of the content-adaptive block-sparse attention library
 * (libsa.so, sm_100a).
 *
 * The library computes causal attention restricted to a content-dependent
 * block-sparse mask:
 *
 *  - the gzip-guided mask M = (M^lit U M^local U I) intersected with the causal
 *    mask, where l_i = 1[r_i > mean(r)] flags blocks whose level-1 compressed
 *    size ratio is above the mean, M^lit_ij = 1[l_i = l_j = 1] and
 *    M^local_ij = 1[|i - j| <= w] in block units, with heads split 50% local
 *    only, 25% literal-long-range only, 25% both ("Gzip-guided sparse
 *    attention: Selecting long-range content by compressibility", Background
 *    and main changes; Core equations);
 *  - the UniGist prefill layout: sink tokens, interleaved gist tokens and a
 *    local window, every token under one unified visibility rule, with gists
 *    shifted to the right end of each tile so that a kernel can skip
 *    non-visible blocks ("UniGist: Towards General and Hardware-aligned
 *    Sequence-level Long Context Compression", Approach);
 *  - gist-scored selective unfolding at decode: the new query is scored
 *    against the gist keys only, the top-k chunks are unfolded to their raw
 *    tokens, and attention runs over gists + unfolded chunks + a local window
 *    ("Simplified Sparse Attention via Gist Tokens", abstract; "Forget, Then
 *    Recall: Learnable Compression and Selective Unfolding via Gist Sparse
 *    Attention", abstract).
 *
 * Conventions shared by every entry point
 *  - Every tensor argument is DEVICE memory owned by the caller. The library
 *    never allocates, frees or synchronises (except sa_get_device_status,
 *    which reads one word back and says so). All work is enqueued on the
 *    caller's stream, in order.
 *  - Arguments are validated on the host before anything is launched; a
 *    failed check returns SA_ERR_INVALID_ARG / SA_ERR_UNSUPPORTED /
 *    SA_ERR_WORKSPACE and touches no device state.
 *  - Strides are in ELEMENTS. The innermost (head_dim) dimension is always
 *    contiguous. Tensors read by TMA need 16-byte aligned base pointers and
 *    strides (bf16: strides multiple of 8 elements).
 *  - Each call that takes a workspace ("ws") needs at least the number of
 *    bytes returned by its *_workspace_size query, 256-byte aligned. The first
 *    word of the workspace is a device status word: kernels that detect a
 *    problem on the device (a bounded wait that ran out, a list longer than
 *    its capacity) set it instead of trapping. The word is cleared by every
 *    call; read it with sa_get_device_status after the stream has finished.
 *  - Launch failures are reported as SA_ERR_CUDA (cudaGetLastError after each
 *    launch).
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* sa_stream_t;

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,  /* bad size, null pointer, misaligned pointer     */
  SA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement   */
  SA_ERR_WORKSPACE = 3,    /* workspace or list capacity too small          */
  SA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed          */
  SA_ERR_TIMEOUT = 5,      /* device status: a bounded wait ran out         */
  SA_ERR_DEVICE = 6,       /* device status: another device-detected fault  */
} sa_status;

typedef enum { SA_MASK_GZIP = 0, SA_MASK_GIST = 1 } sa_mask_kind;

/* Head classes of the gzip mask (Background and main changes). */
typedef enum {
  SA_CLASS_LOCAL = 0,    /* M^local (which contains I)   */
  SA_CLASS_LITERAL = 1,  /* M^lit U I                    */
  SA_CLASS_HYBRID = 2,   /* M^lit U M^local U I          */
} sa_head_class;

typedef enum { SA_DTYPE_BF16 = 0, SA_DTYPE_FP32 = 1 } sa_dtype;

/* Kind of a (query tile, key tile) entry of the tile lists. */
typedef enum {
  SA_TILE_FULL = 0,    /* every pair of the 128x128 tile block is visible     */
  SA_TILE_MASKED = 1,  /* some pairs are not: apply the element mask          */
  SA_TILE_TAIL = 2,    /* gist mode: visible columns lie in the key tile's
                          last gist_tail columns (the shifted gists)          */
} sa_tile_kind;

/* Query/key tile height used by the tile lists and the attention kernels. */
#define SA_TILE 128

/* Mask / layout description.
 *  kind        SA_MASK_GZIP or SA_MASK_GIST.
 *  batch       gzip: number of sequences (each has its own literal flags).
 *              gist: must be 1 - the layout is shared by every batch row.
 *  seq_len     N, tokens (gzip) or positions including gists (gist).
 *  block_size  gzip: b, tokens per block, N % b == 0, and either b % 128 == 0
 *              or 128 % b == 0. gist: 0 for the fine (interleaved) layout; L > 0
 *              for the segment-wise coarse layout of "A Silver Bullet or a
 *              Compromise for Full Attention? ..." (sections 2 and 6): after the
 *              sinks, segments of L raw tokens followed by L / gist_ratio gists
 *              (L % gist_ratio == 0), and query i sees the sinks, the gists not
 *              in its future and every position of its own segment up to i.
 *              The coarse layout takes no explicit flags.
 *  window      gzip: w in BLOCKS (key block j is local to i iff i - j <= w).
 *              gist, fine layout: W >= 1 in POSITIONS (key j is in the window
 *              of i iff i - j < W). gist, coarse layout: ignored.
 *  num_heads   number of query heads H.
 *  head_class  gzip: HOST array [H] of sa_head_class, or NULL for the default
 *              split floor(H/2) local, floor(H/4) literal, rest hybrid, in
 *              that head order. gist: ignored.
 *  sinks       gist: positions [0, sinks) are sink tokens visible to all.
 *  gist_ratio  gist: raw tokens per gist; fine layout: after the sinks a gist
 *              follows every gist_ratio raw tokens (used when no explicit
 *              flags are given).
 *  gist_tail   gist: width of the tail sub-block that holds a tile's gists
 *              after the shift (multiple of 16, <= 128; 0 means 32).
 */
typedef struct sa_mask_desc {
  int32_t kind;
  int32_t batch;
  int64_t seq_len;
  int32_t block_size;
  int32_t window;
  int32_t num_heads;
  int32_t sinks;
  int32_t gist_ratio;
  int32_t gist_tail;
  const int8_t* head_class;
} sa_mask_desc;

/* Literal flags computed on the device from raw bytes: an ESTIMATE of the
 * gzip-based flags ("Gzip-guided sparse attention ...", Core equations: block
 * i is literal iff its compression ratio exceeds the mean). Each block's size
 * c_i comes from a plain DEFLATE encoder of RFC 1951, not from zlib: greedy
 * LZ77 whose candidate at p is the most recent earlier position with the same
 * three bytes that the section-4 table holds in its fast form (every position
 * the parse stops at, and the inside of matches of at most 4 bytes); one
 * final block of the smallest of the fixed-code (section 3.2.6), dynamic-code
 * (section 3.2.7) and stored (section 3.2.4) types; c_i = ceil(bits / 8). On
 * the workloads' bytes the flags equal zlib level 1's, but c_i and the flags
 * can differ from gzip's elsewhere near the mean. Then flags[i] = c_i * B >
 * sum_j c_j.
 *  bytes        DEVICE uint8 [batch, n_bytes]
 *  block_bytes  b, 1 <= b <= 1024, n_bytes % b == 0, B = n_bytes / b
 *  sizes        DEVICE uint32 [batch, B] out: c_i
 *  flags        DEVICE uint8 [batch, B] out: the literal flags, ready for
 *               sa_build_block_mask.
 * Two launches on `stream`; no workspace. */
sa_status sa_literal_flags_device(const uint8_t* bytes, int32_t batch, int64_t n_bytes,
                                  int32_t block_bytes, uint32_t* sizes, uint8_t* flags,
                                  sa_stream_t stream);

/* Output of sa_build_block_mask. All pointers are caller-owned DEVICE memory
 * sized from sa_block_lists_capacity. Unused members may be NULL.
 *
 * Block level (gzip only; B = N / b; one (batch, class) pair at a time,
 * class c in 0..2, index bc = batch * 3 + c):
 *  row_ptr  int32 [batch*3*(B+1)]: query block i of pair bc lists key blocks
 *           col_idx[row_ptr[bc*(B+1)+i] .. row_ptr[bc*(B+1)+i+1]), ascending.
 *           Offsets are absolute; pair bc's entries start at bc * B(B+1)/2.
 *  col_idx  int32 [cap_nnz]
 *  col_ptr  int32 [batch*3*(B+1)]: the transpose (key block -> ascending query
 *           blocks), same offset convention, into row_idx.
 *  row_idx  int32 [cap_nnz]
 *  bits     uint32 [batch*3*B*ceil(B/32)]: row i of pair bc, word k holds bit
 *           (j - 32k) for key block j.
 *
 * Tile level (both kinds; T = ceil(N / 128); gzip: one list per (batch,
 * class); gist: one list): for query tile I, the key tiles J holding at least
 * one visible pair, ascending, with their sa_tile_kind.
 *  tile_row_ptr  int32 [lists*(T+1)], absolute, list l starts at l*T(T+1)/2.
 *  tile_col      int32 [cap_tile_nnz]
 *  tile_kind     int8  [cap_tile_nnz]
 *  tile_col_ptr  int32 [lists*(T+1)]: transpose (key tile -> query tiles).
 *  tile_row      int32 [cap_tile_nnz]
 *  tile_kind_t   int8  [cap_tile_nnz]: kind of each transposed entry.
 *
 * Gist layout (gist only):
 *  perm       int32 [N]: physical index -> logical position (the shift: in
 *             every 128-position tile raw tokens first, then gists, each in
 *             order).
 *  gist_bits  uint32 [ceil(N/32)]: bit p%32 of word p/32 is 1 iff LOGICAL
 *             position p is a gist.
 *  far_idx    int32 [N]: the keys every later query sees whatever its window
 *             (sinks and gists), in logical order, as PHYSICAL indices.
 *  far_ptr    int32 [T+1]: far_ptr[J] = number of those keys at logical
 *             positions below 128*J. Query tile I's window (segment) cannot
 *             reach below key tile Jlo = max(0, I - ceil((W-1)/128)) (coarse:
 *             the tile holding the start of the segment of position 128*I, or
 *             I while that position is a sink), so the keys it sees there are
 *             exactly far_idx[0 .. far_ptr[Jlo]).
 */
typedef struct sa_block_lists {
  int32_t* row_ptr;
  int32_t* col_idx;
  int32_t* col_ptr;
  int32_t* row_idx;
  uint32_t* bits;
  int32_t* tile_row_ptr;
  int32_t* tile_col;
  int8_t* tile_kind;
  int32_t* tile_col_ptr;
  int32_t* tile_row;
  int8_t* tile_kind_t;
  int32_t* perm;
  uint32_t* gist_bits;
  int32_t* far_idx;
  int32_t* far_ptr;
  int64_t cap_nnz;       /* elements of col_idx and row_idx      */
  int64_t cap_tile_nnz;  /* elements of tile_col/_kind/_row/_kind_t */
} sa_block_lists;

/* Element counts each sa_block_lists member needs (0 = not used). */
typedef struct sa_block_lists_sizes {
  int64_t row_ptr, nnz, bits;
  int64_t tile_row_ptr, tile_nnz;
  int64_t perm, gist_bits, far_idx, far_ptr;
} sa_block_lists_sizes;

/* Attention shapes.
 *  dtype        SA_DTYPE_BF16 or SA_DTYPE_FP32; q, k, v, o (and dO) share it.
 *  batch, seq_len       Bt and N; must equal the mask's (gist: any batch).
 *  num_q_heads, num_kv_heads   Hq and Hkv, Hq % Hkv == 0; query head h reads
 *               key/value head h / (Hq / Hkv) (grouped-query attention).
 *  head_dim     d: bf16 64 or 128; fp32 32, 64 or 128.
 *  *_strides    [batch, seq, head] element strides of q, k, v, o; the
 *               head_dim axis is contiguous. LSE is always a dense fp32
 *               [Bt, Hq, N] array.
 *  softmax_scale  0 selects 1/sqrt(d). Scores are q.k * scale; LSE uses the
 *               natural log.
 *  impl         SA_IMPL_AUTO picks the tensor-core kernels when dtype is bf16,
 *               head_dim is 64 or 128, every base pointer is 16-byte aligned
 *               and every stride is a multiple of 8 elements (TMA); otherwise
 *               the CUDA-core kernels. SA_IMPL_TENSOR_CORES on an input that
 *               does not meet those conditions returns SA_ERR_UNSUPPORTED.
 */
typedef enum {
  SA_IMPL_AUTO = 0,
  SA_IMPL_CUDA_CORES = 1,    /* fp32 FMA path (fp32 or bf16 inputs) */
  SA_IMPL_TENSOR_CORES = 2,  /* tcgen05 + TMA path (bf16 only)      */
} sa_impl;

typedef struct sa_attn_desc {
  int32_t dtype;
  int32_t batch;
  int64_t seq_len;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  float softmax_scale;
  int64_t q_strides[3];
  int64_t k_strides[3];
  int64_t v_strides[3];
  int64_t o_strides[3];
  int32_t impl;
} sa_attn_desc;

/* Chunk selection at decode (one selection per KV group).
 *  SUM_LOGITS_PER_GROUP  top_k chunks by the sum over the group's query heads
 *                        of q_h . gist_k * scale.
 *  SUM_PROBS_PER_GROUP   top_k chunks by the sum over the group's query heads
 *                        of each head's softmax over all the group's gists.
 *  TOP_P_PER_GROUP       the group's summed logits, softmax over the eligible
 *                        chunks: the smallest score-ordered prefix whose
 *                        probability reaches top_p, at most top_k chunks.
 *  TOP_K_PER_HEAD        every query head takes the top_k chunks of its own
 *                        q_h . gist_k * scale and attends over its own chunks
 *                        (sel is then [n_seq, Hq, top_k]).
 * Ties go to the lower chunk index in every rule. The pages of "Simplified
 * Sparse Attention via Gist Tokens" name a top-k and a top-p selection from
 * logits and a per-group selection; the three readings above are this
 * library's. */
typedef enum {
  SA_SELECT_SUM_LOGITS_PER_GROUP = 0,
  SA_SELECT_SUM_PROBS_PER_GROUP = 1,
  SA_SELECT_TOP_P_PER_GROUP = 2,
  SA_SELECT_TOP_K_PER_HEAD = 3
} sa_select_rule;

/* Decode shapes (one new query token per sequence).
 *  q          [n_seq, Hq, d]            strides q_strides {seq, head}
 *  gist_k/v   [n_seq, Hkv, n_gists, d]  strides gist_strides {seq, head, gist}
 *  k/v_cache  [n_seq, Hkv, cache_len, d] strides cache_strides {seq, head, pos}
 *  o          [n_seq, Hq, d]            strides o_strides {seq, head}
 *  lse        fp32 [n_seq, Hq] dense
 *  sel        int32 [n_seq, Hkv, top_k] dense ([n_seq, Hq, top_k] under
 *             SA_SELECT_TOP_K_PER_HEAD): the selected chunk indices,
 *             ascending, -1 padded when fewer chunks are eligible.
 *  chunk      raw tokens per gist; n_gists * chunk == cache_len.
 *  window     the last `window` cache positions are always attended; a chunk
 *             is eligible for selection iff it lies entirely before them.
 *  top_k      chunks unfolded per (sequence, KV head), 0 <= top_k <= 256.
 *  select_rule  an sa_select_rule (see above).
 *  top_p      TOP_P_PER_GROUP only: 0 < top_p <= 1.
 * All bf16; head_dim 128; Hq / Hkv <= 8.
 */
typedef struct sa_decode_desc {
  int32_t n_seq;
  int32_t cache_len;
  int32_t chunk;
  int32_t n_gists;
  int32_t top_k;
  int32_t window;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t select_rule;
  float softmax_scale;
  int64_t q_strides[2];
  int64_t gist_strides[3];
  int64_t cache_strides[3];
  int64_t o_strides[2];
  float top_p;
} sa_decode_desc;

/* Gist-of-gist decode shapes ("Forget, Then Recall: ... Gist Sparse
 * Attention", abstract: recursive gist-of-gist construction for
 * multi-resolution access with logarithmic per-step cost; the level structure
 * below is this library's reading). Level 1 has one gist per `chunk` raw
 * tokens (n_gists of them), level 2 one gist per `fanout` consecutive level-1
 * gists (n_gists / fanout of them, a "group").
 *  q           [n_seq, Hq, d]                   strides q_strides {seq, head}
 *  gist2_k/v   [n_seq, Hkv, n_gists/fanout, d]  strides gist2_strides
 *  gist_k/v    [n_seq, Hkv, n_gists, d]         strides gist_strides
 *  k/v_cache   [n_seq, Hkv, cache_len, d]       strides cache_strides
 *  o, lse      as for sa_gist_decode.
 *  sel_groups  int32 [n_seq, Hkv, top_k2]: kept groups, ascending, -1 padded.
 *  sel_chunks  int32 [n_seq, Hkv, top_k]: unfolded chunks, ascending, -1 padded.
 * Per (sequence, KV group): the top_k2 groups wholly before the window by the
 * summed logit of their level-2 gist, then the top_k chunks among those
 * groups' level-1 gists by the same score (ties to the lower index); every
 * head attends in one softmax over all level-2 gists, the kept groups'
 * level-1 gists, the unfolded chunks' raw tokens and the last `window` raw
 * tokens. All bf16, head_dim 128, Hq / Hkv in {1, 2, 4, 8}; n_gists % fanout
 * == 0, n_gists * chunk == cache_len, top_k2, top_k <= 256, n_gists / fanout
 * and top_k2 * fanout <= 8192. K and V of a level share strides. */
typedef struct sa_hier_decode_desc {
  int32_t n_seq;
  int32_t cache_len;
  int32_t chunk;
  int32_t n_gists;
  int32_t fanout;
  int32_t top_k2;
  int32_t top_k;
  int32_t window;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  float softmax_scale;
  int64_t q_strides[2];
  int64_t gist_strides[3];
  int64_t gist2_strides[3];
  int64_t cache_strides[3];
  int64_t o_strides[2];
} sa_hier_decode_desc;

sa_status sa_gist_hier_decode_workspace_size(const sa_hier_decode_desc* desc, size_t* bytes);

/* One gist-of-gist decode step (CUDA cores: level-2 pass, group selection,
 * level-1 pass over the kept groups, chunk selection, raw pass, combine). */
sa_status sa_gist_hier_decode(const sa_hier_decode_desc* desc, const void* q,
                              const void* gist2_k, const void* gist2_v, const void* gist_k,
                              const void* gist_v, const void* k_cache, const void* v_cache,
                              int32_t* sel_groups, int32_t* sel_chunks, void* o, float* lse,
                              void* ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------------ misc */

/* Library version string, e.g. "0.1.0 (sm_100a)". Never NULL. */
const char* sa_version(void);

/* Human-readable name of a status code. Never NULL. */
const char* sa_status_string(sa_status st);

/* Reads the device status word at the start of a workspace used by an
 * earlier call: copies it to *out on `stream` and synchronises that stream
 * (the only call of this library that blocks). SA_OK, SA_ERR_TIMEOUT or
 * SA_ERR_DEVICE. ws == NULL reads the status word of the fixed scratch array
 * of sa_gist_decode_noalloc on the current device instead. */
sa_status sa_get_device_status(const void* ws, sa_stream_t stream, sa_status* out);

/* Literal flags from per-block compressed sizes (HOST helper, no CUDA).
 * r_i = sizes[i] / b and the mean ratio share the divisor b, so the flag
 * l_i = 1[r_i > mean(r)] ("Gzip-guided sparse attention ...", Core equations)
 * is evaluated exactly as sizes[i] * B > sum(sizes) in 64-bit integers.
 * sizes: host [B]; flags: host [B] (0/1). B >= 1. */
sa_status sa_literal_flags_from_sizes(const uint32_t* sizes, int32_t num_blocks,
                                      uint8_t* flags);

/* -------------------------------------------------------- mask builder */

/* Capacities of every sa_block_lists member for a description. */
sa_status sa_block_lists_capacity(const sa_mask_desc* desc,
                                  sa_block_lists_sizes* out);

/* Bytes of workspace sa_build_block_mask needs. */
sa_status sa_build_block_mask_workspace_size(const sa_mask_desc* desc, size_t* bytes);

/* Builds the block and tile lists on the GPU.
 * Defined by "Gzip-guided sparse attention: Selecting long-range content by
 * compressibility" (Core equations: M = (M^lit U M^local U I) intersected with
 * the causal mask, per head class) and "UniGist: Towards General and
 * Hardware-aligned Sequence-level Long Context Compression" (Approach: sinks,
 * gists and a local window under one rule; gists shifted to each tile's end).
 *  d_flags  gzip: DEVICE uint8 [batch, B] literal flags (0/1), e.g. from
 *           sa_literal_flags_from_sizes. gist: DEVICE uint8 [N] with 1 for
 *           the LOGICAL positions that are gists, or NULL for the regular
 *           pattern (sinks, then one gist after every gist_ratio raw tokens;
 *           coarse layout: NULL only, its segments as block_size states).
 *  out      lists to fill; capacities checked against sa_block_lists_capacity.
 * Bit-exact: the lists depend only on integers. */
sa_status sa_build_block_mask(const sa_mask_desc* desc, const uint8_t* d_flags,
                              const sa_block_lists* out, void* ws, size_t ws_bytes,
                              sa_stream_t stream);

/* --------------------------------------------------------- attention */

sa_status sa_forward_workspace_size(const sa_attn_desc* attn, const sa_mask_desc* mask,
                                    size_t* bytes);

/* O and LSE of causal attention restricted to the mask ("Gzip-guided sparse
 * attention ...", Core equations: attention sees only the mask's blocks;
 * Scope: skipping the masked blocks is what turns sparsity into speed;
 * "UniGist ...", Approach: kernels skip the blocks no query of a tile sees).
 * For every query row
 * p: s_pq = q_p . k_q * scale over the keys q the mask allows,
 * LSE_p = log sum_q exp(s_pq), O_p = sum_q exp(s_pq - LSE_p) v_q.
 * Only key tiles listed in `lists` are read. Gist mode takes q, k, v, o and
 * lse in PHYSICAL (shifted) order, as given by lists->perm.
 *  q [Bt, N, Hq, d], k/v [Bt, N, Hkv, d], o [Bt, N, Hq, d] (dtype of attn),
 *  lse fp32 [Bt, Hq, N]. */
sa_status sa_forward(const sa_attn_desc* attn, const sa_mask_desc* mask,
                     const void* q, const void* k, const void* v,
                     const sa_block_lists* lists, void* o, float* lse,
                     void* ws, size_t ws_bytes, sa_stream_t stream);

sa_status sa_backward_workspace_size(const sa_attn_desc* attn, const sa_mask_desc* mask,
                                     size_t* bytes);

/* Gradients of the forward for an upstream dO ("UniGist ...", Approach:
 * one-pass training under the same sparse pattern, measured by forward and
 * backward latency), same layout/strides as o:
 * D_p = sum dO_p * O_p, P = exp(s - LSE), dV = P^T dO, dP = dO V^T,
 * dS = P * (dP - D), dQ = dS K * scale, dK = dS^T Q * scale.
 * o and lse must come from sa_forward with the same inputs.
 * dq fp32 dense [Bt, N, Hq, d]; dk, dv fp32 dense [Bt, N, Hkv, d] (summed over
 * the query heads of a group). The tensor-core path (bf16, d 64 or 128, gzip
 * masks or the gist layout) runs two passes: a query-major one for dQ (S and dP
 * recomputed, dQ written once per row, no float atomics) and a key-major one
 * for dK and dV; gist mode adds the far-key contributions of every sink and
 * gist in a last scatter. Deterministic: the same inputs give the same bits. */
sa_status sa_backward(const sa_attn_desc* attn, const sa_mask_desc* mask,
                      const void* q, const void* k, const void* v,
                      const void* o, const float* lse, const void* dout,
                      const sa_block_lists* lists, float* dq, float* dk, float* dv,
                      void* ws, size_t ws_bytes, sa_stream_t stream);

/* ------------------------------------------------------------ decode */

sa_status sa_gist_decode_workspace_size(const sa_decode_desc* desc, size_t* bytes);

/* One decode step: gist scores -> per-group top-k -> attention over
 * {all gists} U {raw tokens of the selected chunks} U {last `window` tokens}
 * ("Simplified Sparse Attention via Gist Tokens", record: score the query
 * against the gists only and unfold the selected chunks; "Forget, Then
 * Recall: ... Gist Sparse Attention", abstract: selective unfolding).
 * Outputs o (bf16), lse (fp32) and the selected chunks. */
sa_status sa_gist_decode(const sa_decode_desc* desc, const void* q,
                         const void* gist_k, const void* gist_v,
                         const void* k_cache, const void* v_cache,
                         int32_t* sel_chunks, void* o, float* lse,
                         void* ws, size_t ws_bytes, sa_stream_t stream);

/* Allocation-free variant of sa_gist_decode (the method's pages have no
 * counterpart; this is a deployment convenience).
 *
 * Some callers cannot allocate device memory: a serving engine that reserves
 * all free memory for its KV cache at start-up and forbids later allocations,
 * a plugin that a host framework only hands raw pointers, or a decode loop
 * in which cudaMalloc's implicit device synchronisation would stall the other
 * streams. This entry point takes the same inputs and outputs as
 * sa_gist_decode but no workspace: its scratch is a fixed 16 MiB array in
 * device memory that every GPU loading the library holds until the process
 * exits. It calls no cudaMalloc or cudaFree.
 *  - Sizes whose workspace (sa_gist_decode_workspace_size) exceeds 16 MiB
 *    return SA_ERR_WORKSPACE; use sa_gist_decode for them.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture. The address is cached per device and context: after
 *    cudaDeviceReset (a new context) the next call looks it up again, so
 *    that call, too, belongs outside a stream capture.
 *  - Every call on a device shares the one array, which keeps the last call's
 *    contents (its status word is cleared by each call). Calls that overlap on
 *    the GPU - on different streams, or from different host threads without
 *    ordering - race on it; serialise them.
 *  - A device-side problem (a bounded wait that ran out) sets the status
 *    word at the start of the array: read it with sa_get_device_status(NULL,
 *    stream, &st) after the call, with the same device current. */
sa_status sa_gist_decode_noalloc(const sa_decode_desc* desc, const void* q,
                                 const void* gist_k, const void* gist_v,
                                 const void* k_cache, const void* v_cache,
                                 int32_t* sel_chunks, void* o, float* lse,
                                 sa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SA_H_ */
