/*
 * nsa.h -- C ABI of the B200 (sm_100a) NSA compressed-attention library.
 *
 * The library computes the compressed branch of Native Sparse Attention:
 *   nsa_compress            sliding-window compression of raw K and V
 *                           ("aclnnNsaCompress", Formula section);
 *   nsa_compress_attention  causal GQA attention over the compressed blocks,
 *                           importance scores, head-group sum and per-query
 *                           top-k of selection blocks
 *                           ("mindspore.ops.nsa_compress_attention", steps 1-7);
 *   nsa_compress_attention_masked  the same with the optional atten_mask /
 *                           topk_mask of the page's keyword arguments
 *   nsa_compress_paged, nsa_compress_attention_paged
 *                           the compression into, and the attention over, a
 *                           paged compressed K/V cache (decode)
 *   nsa_select_attention    attention over the raw K/V blocks that top-k lists
 *                           ("lite_boost.ops.rain_fusion_attention");
 *   nsa_compress_attention_backward, nsa_compress_backward
 *                           gradients of the compressed attention and of the
 *                           compression (training scenario).
 *
 * Conventions shared by every entry point
 *   - Layout is TND ("mindspore.ops.nsa_compress_attention", note list):
 *     a tensor (T, N, D) is row-major, D contiguous, then heads, then the
 *     concatenated tokens of all sequences of the batch.
 *   - Sequence lengths are HOST int32 arrays of `batch` cumulative ends
 *     (prefix sums, no leading 0, non-decreasing), as the pages require
 *     ("cumulative sum mode" on the aclnnNsaCompress page; "prefix-sum mode"
 *     for actual_seq_qlen / actual_cmp_seq_kvlen / actual_sel_seq_kvlen).
 *   - Tensor pointers are DEVICE pointers, 16-byte aligned, owned by the
 *     caller.  The library allocates no memory and keeps no state between
 *     calls (the one exception is the fixed scratch array behind
 *     nsa_compress_attention_noalloc, declared at the end of this file).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; argument errors are returned
 *     synchronously before anything is enqueued ("aclnnNsaCompress": the
 *     first phase validates the parameters and returns a status code).
 *   - Results are deterministic: two calls with the same inputs produce
 *     bitwise-identical outputs ("aclnnNsaCompress", deterministic
 *     computation by default).  No atomics on any result.
 */
#ifndef NSA_B200_H
#define NSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NSA_OK = 0,
    NSA_ERR_INVALID_ARG = 1,   /* a value, pointer or size breaks a stated constraint */
    NSA_ERR_UNSUPPORTED = 2,   /* valid per the pages but outside what this build runs */
    NSA_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small           */
    NSA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed           */
    NSA_ERR_TIMEOUT = 5        /* a device-side wait gave up (reported after the fact) */
} nsa_status_t;

typedef enum { NSA_BF16 = 0, NSA_FP16 = 1 } nsa_dtype_t;

/* Human-readable name of a status code.  Never NULL; static storage. */
const char* nsa_status_string(nsa_status_t status);

/*
 * Number of compressed blocks per sequence ("aclnnNsaCompress", Formula
 * section: block i exists for 0 <= i <= floor((S - l)/d); a sequence with
 * S < l has none).
 *   cu_seqlens  host, [batch] cumulative raw lengths
 *   cu_cmp_out  host, [batch] written with the cumulative compressed lengths
 *   total_out   host, optional (may be NULL): total compressed rows Tc
 * Errors: NSA_ERR_INVALID_ARG for NULL arrays, batch < 1, l or d < 1, or
 * decreasing prefix sums.  Pure host function, no CUDA call.
 */
nsa_status_t nsa_compress_out_len(const int32_t* cu_seqlens, int batch, int l, int d,
                                  int32_t* cu_cmp_out, int64_t* total_out);

/*
 * Sliding-window compression of K and V ("aclnnNsaCompress", Formula
 * section), with phi read as the weighted sum over the window:
 *   kcmp[c0+i, n, :] = sum_{j<l} w[j, n] * k[s0 + i*d + j, n, :]
 *   vcmp[c0+i, n, :] = sum_{j<l} w[j, n] * v[s0 + i*d + j, n, :]
 * for every sequence (raw rows start at s0, compressed rows at c0) and every
 * i < n_cmp.  fp32 accumulation in window order, one rounding (RNE) to dtype.
 *   k     device (T2, N2, D1), dtype        v     device (T2, N2, D2), dtype
 *   w     device (l, N2), dtype: one weight per window position and head,
 *         shared by K and V and by every head dimension
 *   kcmp  device (Tc, N2, D1), written      vcmp  device (Tc, N2, D2), written
 *   Tc = total of nsa_compress_out_len.  v/vcmp may both be NULL (K only).
 * Constraints (NSA_ERR_INVALID_ARG): l, d multiples of 16; 16 <= d <= l <= 128
 * ("select/compress" constraint list of mindspore.ops.nsa_compress_attention);
 * D1, D2 multiples of 16 and <= 256 (aclnnNsaCompress constraint list);
 * N2 >= 1; pointers 16-byte aligned.
 */
nsa_status_t nsa_compress(const void* k, const void* v, const void* w, int l, int d,
                          const int32_t* cu_seqlens, int batch, int n2, int d1, int d2,
                          nsa_dtype_t dtype, void* kcmp, void* vcmp, void* stream);

/*
 * nsa_compress into a paged compressed cache: block i of sequence b goes to row
 * i % page_size of pool page block_table[b * max_pages_per_seq + i / page_size].
 * Only blocks first_block[b] .. n_cmp_b - 1 are computed (first_block NULL: all),
 * so a decode step compresses just the window its new token completed
 * (first_block[b] = n_cmp_b - 1 when (S_b - l) % d == 0, else n_cmp_b) and
 * nsa_compress_attention_paged then reads the cache.  Same arithmetic as
 * nsa_compress (bitwise equal rows).
 *   kcmp_pages, vcmp_pages  device (num_pages, page_size, N2, D1 / D2), written
 *   block_table   device int32 (batch, max_pages_per_seq); an entry outside
 *                 [0, num_pages) is never written through: the store is skipped
 *                 and nsa_compress_status reports NSA_ERR_INVALID_ARG
 *   first_block   host int32 [batch] or NULL; 0 <= first_block[b] <= n_cmp_b
 * Other arguments and constraints as nsa_compress; a block table row too short
 * for a sequence's blocks is NSA_ERR_INVALID_ARG.
 */
nsa_status_t nsa_compress_paged(const void* k, const void* v, const void* w, int l, int d,
                                const int32_t* cu_seqlens, int batch, int n2, int d1, int d2,
                                nsa_dtype_t dtype, void* kcmp_pages, void* vcmp_pages, int64_t num_pages,
                                int page_size, const int32_t* block_table, int max_pages_per_seq,
                                const int32_t* first_block, void* stream);

/*
 * Workspace bytes that nsa_compress_attention needs for these arguments.
 * Same argument meaning as nsa_compress_attention.  Pure host function.
 */
nsa_status_t nsa_compress_attention_workspace_size(
    int head_num, int n2, int d1, int d2, int l, int d, int lp, int count,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
    int batch, size_t* bytes);

/*
 * Compressed attention with importance scores and top-k
 * ("mindspore.ops.nsa_compress_attention", steps 1-7; returns list).
 * Per sequence b, query row t_loc sits at position t = t_loc + off_b with
 * off_b = max(0, (n_cmp_b - 1)*d + l - S_q_b) (0 when n_cmp_b = 0); compressed
 * block i is visible iff i*d + l - 1 <= t.  For head h of KV group g = h / G
 * (G = head_num / n2):
 *   s_i = scale * q[t,h,:] . kcmp[i,g,:]        (step 1)
 *   P_i = exp(s_i - m) / L,  m = max s, L = sum exp(s - m)   (step 2)
 *   out[t,h,:] = sum_i P_i vcmp[i,g,:]          (step 3)
 *   P_slc[j] = sum_{m<l'/d} sum_{n<l/d} P[l'/d*j - m - n]   (step 4)
 *   P_slc'[t,g,j] = sum over the G heads of group g          (step 5)
 *   topk_indices[t,g,:] = the min(count, #candidates) largest P_slc' over
 *     the candidates j < n_sel_b with j*l' <= t, ties to the smaller j,
 *     listed ascending, then -1 padding (step 7; index convention of
 *     lite_boost.ops.rain_fusion_attention select_idx).
 * A row that sees no block gets out = 0, softmax_max = -inf, softmax_sum = 0
 * and all indices -1.
 * Arguments
 *   q         device (T1, N1, D1) dtype      kcmp  device (Tc, N2, D1) dtype
 *   vcmp      device (Tc, N2, D2) dtype      scale scale_value of step 1
 *   head_num  N1 (== number of query heads)
 *   l, d, lp, count  compress_block_size, compress_stride, select_block_size,
 *             select_block_count
 *   cu_seqlens_q, cu_cmp_kv, cu_sel_kv  host [batch] prefix sums
 *   attention_out device (T1, N1, D2) dtype     topk_indices device (T1, N2, count) int32
 *   softmax_max, softmax_sum  device (T1, N1, 8) fp32, 8 equal copies;
 *             max of the scaled scores and sum of exp(s - max) (natural exp)
 *   workspace device, >= nsa_compress_attention_workspace_size bytes,
 *             256-byte aligned; its first 16 bytes receive a device error
 *             word read by nsa_workspace_status
 * Constraints (NSA_ERR_INVALID_ARG, from the note list of
 * mindspore.ops.nsa_compress_attention): l, d, lp multiples of 16;
 * 16 <= l <= 128; 16 <= d <= 64; 16 <= lp <= 128; l >= d; lp >= l; lp % d == 0;
 * 1 <= count <= 32; D1 >= D2; D1, D2 multiples of 16; N1 >= N2, N1 % N2 == 0.
 * NSA_ERR_UNSUPPORTED: l % d != 0 (the importance sum needs integer l/d),
 * D1 or D2 > 256, more than 128 query heads per KV group, or shapes whose
 * on-chip tiles do not fit one SM.
 */
nsa_status_t nsa_compress_attention(
    const void* q, const void* kcmp, const void* vcmp, float scale, int head_num,
    int l, int d, int lp, int count,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
    int batch, int n2, int d1, int d2, nsa_dtype_t dtype,
    void* attention_out, int32_t* topk_indices, float* softmax_max, float* softmax_sum,
    void* workspace, size_t workspace_bytes, void* stream);

/*
 * nsa_compress_attention with the page's optional keyword arguments
 * ("mindspore.ops.nsa_compress_attention": atten_mask, shape (S1, S2) with S2
 * the compressed KV length, applied to QK in step 1; topk_mask, shape
 * (S1, S2) with S2 the select KV length, applied to P'_slc in step 6; dtype
 * bool).  Reading of the page, which leaves both open: a non-zero byte at
 * (row, block) removes that pair -- the block from the visible set of the
 * row, or the selection block from its top-k candidates; one matrix serves
 * every sequence of the batch and every head, and its row is the query's
 * index inside its sequence (0 .. S_q-1).  The masks act on top of the
 * built-in causal rules; a row left without an attended block is an empty
 * row (zeros, max -inf, sum 0, indices -1).
 *   atten_mask  device bytes, row-major, am_rows x am_cols (row stride
 *               am_cols); NULL = no mask.  Needs am_rows >= every S_q and
 *               am_cols >= every sequence's compressed block count.
 *   topk_mask   device bytes, tm_rows x tm_cols, NULL = no mask.  Needs
 *               tm_rows >= every S_q and tm_cols >= every n_sel.
 * The call first packs each given mask into bit rows inside the workspace
 * (one launch per mask), so the attention kernel reads 1 bit per (row,
 * block).  Workspace: nsa_compress_attention_masked_workspace_size with the
 * same masks present.  Other arguments, outputs and errors as
 * nsa_compress_attention; a mask too small for the batch is
 * NSA_ERR_INVALID_ARG.  With both masks NULL the call is
 * nsa_compress_attention.
 */
/*
 * nsa_compress_attention over a paged compressed K/V cache (the block_table of
 * "lite_boost.ops.rain_fusion_attention", applied to the compressed blocks):
 * sequence b's compressed block i lives in row i % page_size of pool page
 * block_table[b * max_pages_per_seq + i / page_size].  The decode shape -- one
 * query per sequence (cu_seqlens_q = 1, 2, ..., batch), which by the query
 * offset of step 1 sits at the last raw position the blocks cover -- is the
 * main use; any query counts are accepted.  Outputs, workspace
 * (nsa_compress_attention_workspace_size with the same arguments) and errors as
 * nsa_compress_attention, whose results it reproduces bit for bit when the
 * pages hold the same rows.
 *   kcmp_pages, vcmp_pages  device (num_pages, page_size, N2, D1 / D2) dtype
 *   block_table   device int32 (batch, max_pages_per_seq), 4-byte aligned.  An
 *                 entry outside [0, num_pages) reads zeros (never faults).
 *   cu_cmp_kv     host prefix sums of the sequences' compressed block counts
 * Rows of a sequence's last page past its block count must hold finite values
 * (they meet zero weights in P . V).  Constraints: page_size a multiple of 8
 * that divides the KV tile (128 blocks when l'/d is 1, 2, 4 or 8; 96, 80 or
 * 112 otherwise) -- NSA_ERR_UNSUPPORTED; a block table row too short for a
 * sequence -- NSA_ERR_INVALID_ARG.
 */
nsa_status_t nsa_compress_attention_paged(
    const void* q, const void* kcmp_pages, const void* vcmp_pages, int64_t num_pages, int page_size,
    const int32_t* block_table, int max_pages_per_seq, float scale, int head_num, int l, int d, int lp,
    int count, const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv, int batch,
    int n2, int d1, int d2, nsa_dtype_t dtype, void* attention_out, int32_t* topk_indices,
    float* softmax_max, float* softmax_sum, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Workspace bytes of nsa_compress_attention_masked: that of the unmasked call
 * plus the bit-packed rows of each mask that is present (with_* non-zero).
 * Pure host function.
 */
nsa_status_t nsa_compress_attention_masked_workspace_size(
    int head_num, int n2, int d1, int d2, int l, int d, int lp, int count,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
    int batch, int with_atten_mask, int with_topk_mask, size_t* bytes);

nsa_status_t nsa_compress_attention_masked(
    const void* q, const void* kcmp, const void* vcmp, float scale, int head_num,
    int l, int d, int lp, int count,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
    int batch, int n2, int d1, int d2, nsa_dtype_t dtype,
    const uint8_t* atten_mask, int am_rows, int am_cols,
    const uint8_t* topk_mask, int tm_rows, int tm_cols,
    void* attention_out, int32_t* topk_indices, float* softmax_max, float* softmax_sum,
    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sharding one problem by KV-head group, with no communication: every
 * (token, KV group) pair of steps 1-7 is independent, and a group's G query
 * heads, its K/V head and its top-k row are read and written by it alone.
 * A rank that computes groups [group_begin, group_begin + group_count) of
 * the problem needs only those heads' data and writes only those outputs.
 *
 * nsa_shard_groups: the balanced contiguous split of n2 groups over `world`
 * ranks (the first n2 % world ranks take one group more).  Pure host
 * function; NSA_ERR_INVALID_ARG for n2 < 1, world < 1, rank outside
 * [0, world) or NULL outputs.
 */
nsa_status_t nsa_shard_groups(int n2, int world, int rank, int* group_begin, int* group_count);

/*
 * Workspace bytes of nsa_compress_attention_shard for these arguments (a
 * shard needs less than the whole problem).  Pure host function.
 */
nsa_status_t nsa_compress_attention_shard_workspace_size(
    int head_num, int n2, int d1, int d2, int l, int d, int lp, int count,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
    int batch, int group_begin, int group_count, size_t* bytes);

/*
 * nsa_compress_attention restricted to the KV groups [group_begin,
 * group_begin + group_count): the query heads h with h / G in that range,
 * their attention_out / softmax_max / softmax_sum rows, and topk_indices
 * [t, g, :] for g in that range.  Tensors are the whole problem's (same
 * shapes and layout as nsa_compress_attention); only the shard's heads are
 * read and only the shard's outputs are written, everything else is left
 * untouched.  The results are bitwise those of nsa_compress_attention for
 * the same heads.  NSA_ERR_INVALID_ARG when the range is not inside [0, n2);
 * other arguments and errors as nsa_compress_attention.
 */
nsa_status_t nsa_compress_attention_shard(
    const void* q, const void* kcmp, const void* vcmp, float scale, int head_num,
    int l, int d, int lp, int count,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
    int batch, int n2, int d1, int d2, nsa_dtype_t dtype, int group_begin, int group_count,
    void* attention_out, int32_t* topk_indices, float* softmax_max, float* softmax_sum,
    void* workspace, size_t workspace_bytes, void* stream);

/*
 * The work items a shard's launch runs, for inspection on the host (no CUDA
 * call): each item is (first query row, tokens, KV group) as three int32 in
 * `items` (capacity items fit); *n_items receives the total.  The items of
 * the shards of nsa_shard_groups cover every (query row, KV group) pair of
 * the problem exactly once.
 */
nsa_status_t nsa_compress_attention_shard_plan(
    int head_num, int n2, int d1, int d2, int l, int d, int lp, int count,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
    int batch, int group_begin, int group_count, int32_t* items, int64_t capacity, int64_t* n_items);

/*
 * Bytes of device workspace nsa_select_attention needs for these shapes
 * (same arguments; a pure host computation).
 */
nsa_status_t nsa_select_attention_workspace_size(
    int head_num, int n2, int d1, int d2, int lp, int count,
    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv, int batch, size_t* bytes);

/*
 * Selection attention: attention over the raw K/V blocks of l' tokens listed
 * per (query row, KV group) -- the consumer of nsa_compress_attention's
 * topk_indices ("lite_boost.ops.rain_fusion_attention": block-sparse
 * attention over index lists that hold ascending valid block indices, then
 * -1 padding; causal mask, mask_type 0; GQA; returns attention_out and
 * softmax_lse).  Query row t_loc of sequence b sits at key position
 * t = t_loc + (S_kv_b - S_q_b); for head h of group g = h / G it attends to
 * the keys p of the blocks listed in topk_indices[t, g, :] (block j holds
 * p = j*lp .. j*lp + lp - 1) with p <= t and p < S_kv_b:
 *   attention_out[t,h,:] = sum_p softmax_p(scale * q[t,h,:] . k[p,g,:]) v[p,g,:]
 *   softmax_lse[t,h]     = log sum_p exp(scale * q . k_p)  (natural log)
 * The list is read as a set: -1 entries, blocks past the end of the
 * sequence and repeats are skipped.  A row that attends to nothing gets
 * attention_out = 0 and softmax_lse = -inf.
 * Arguments
 *   q             device (T1, N1, D1) dtype      k device (T2, N2, D1) dtype
 *   v             device (T2, N2, D2) dtype
 *   topk_indices  device (T1, N2, count) int32 (as written by nsa_compress_attention)
 *   scale, head_num (N1), lp (block size l'), count (entries per list)
 *   cu_seqlens_q, cu_seqlens_kv  host [batch] prefix sums (no leading 0)
 *   attention_out device (T1, N1, D2) dtype      softmax_lse device (T1, N1) fp32
 *   workspace     device, >= nsa_select_attention_workspace_size bytes,
 *                 256-byte aligned; its first 16 bytes receive the device error
 *                 word read by nsa_workspace_status
 * Constraints: lp a multiple of 16 in [16, 128]; 1 <= count <= 32; D1, D2
 * multiples of 16; topk_indices and softmax_lse 4-byte aligned, the other
 * tensors 16-byte aligned (NSA_ERR_INVALID_ARG); D1 or D2 > 256, more than
 * 128 query heads per KV group, or a sequence of more than 819200 blocks of
 * lp keys (NSA_ERR_UNSUPPORTED).  Two launches on `stream`: a planning kernel
 * that gathers each tile's union of listed blocks, then the attention kernel.
 */
nsa_status_t nsa_select_attention(
    const void* q, const void* k, const void* v, const int32_t* topk_indices, float scale,
    int head_num, int lp, int count, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv,
    int batch, int n2, int d1, int d2, nsa_dtype_t dtype,
    void* attention_out, float* softmax_lse, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Bytes of device workspace nsa_compress_attention_backward needs (a pure
 * host computation; same shape arguments as the backward call).
 */
nsa_status_t nsa_compress_attention_backward_workspace_size(
    int head_num, int n2, int d1, int d2, int l, int d,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, int batch, size_t* bytes);

/*
 * Gradient of attention_out of nsa_compress_attention (its steps 1-3) with
 * respect to q, kcmp and vcmp.  The page returns softmax_max / softmax_sum
 * for gradient back-propagation ("mindspore.ops.nsa_compress_attention",
 * Returns) and prints no backward formulas; they follow from the forward
 * definition, with P_i = exp(s_i - m) / L over the visible blocks:
 *   dvcmp_i = sum over rows and the G heads of group g of P_i dout
 *   dS_i    = P_i (dout . vcmp_i - dout . attention_out)
 *   dq      = scale sum_i dS_i kcmp_i
 *   dkcmp_i = scale sum over rows and heads of dS_i q
 * The importance scores and topk_indices are index outputs: no gradient.
 * Arguments
 *   q, kcmp, vcmp      the forward's inputs (device, TND, dtype)
 *   attention_out      device (T1, N1, D2) dtype, the forward's output
 *   dout               device (T1, N1, D2) dtype, gradient of attention_out
 *   softmax_max, softmax_sum  device (T1, N1, 8) fp32, the forward's statistics
 *   scale, head_num, l, d, cu_seqlens_q, cu_cmp_kv, batch, n2, d1, d2, dtype
 *                      as in the forward call
 *   dq                 device (T1, N1, D1) fp32, overwritten
 *   dkcmp, dvcmp       device (Tc, N2, D1) / (Tc, N2, D2) fp32, overwritten
 *   workspace          device, >= the size above, 256-byte aligned; first 16
 *                      bytes: error word (nsa_workspace_status)
 * Constraints: those of the forward without lp / count, and
 * ceil(D1/64) + ceil(D2/64) <= 6 (Q, dO, K, V tiles on chip together:
 * NSA_ERR_UNSUPPORTED beyond).  No atten_mask.  Deterministic: each dkcmp /
 * dvcmp row is the sum of per-run partials in a fixed order, no atomics.
 * Launches on `stream`: statistics prep, dq, dkcmp/dvcmp runs (one launch,
 * or two when D2 > 128), partial reduction.
 */
nsa_status_t nsa_compress_attention_backward(
    const void* q, const void* kcmp, const void* vcmp, const void* attention_out, const void* dout,
    const float* softmax_max, const float* softmax_sum, float scale, int head_num, int l, int d,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, int batch, int n2, int d1, int d2,
    nsa_dtype_t dtype, float* dq, float* dkcmp, float* dvcmp, void* workspace, size_t workspace_bytes,
    void* stream);

/*
 * Bytes of device workspace nsa_compress_backward needs (host computation): a
 * header, one int per compressed row and 4 MiB for the dw partial sums.
 */
nsa_status_t nsa_compress_backward_workspace_size(const int32_t* cu_seqlens, int batch, int l, int d,
                                                  size_t* bytes);

/*
 * Gradient of nsa_compress ("aclnnNsaCompress", Formula: kcmp_i = sum_j
 * w[j] k[i d + j], per head; training scenario).  The compression is linear:
 *   dk[p]   = sum over the windows i that cover p of w[p - i d] dkcmp_i
 *   dw[j,n] = sum_i dkcmp_i . k[i d + j] + dvcmp_i . v[i d + j]   (one w for K and V)
 * Raw rows that no window covers get dk = 0.
 * Arguments
 *   k, v, w            the forward's inputs (device; v may be NULL, then dvcmp and dv too)
 *   dkcmp, dvcmp       device (Tc, N2, D1) / (Tc, N2, D2) fp32, incoming gradients
 *   dk, dv             device (T, N2, D1) / (T, N2, D2) fp32, overwritten
 *   dw                 device (l, N2) fp32, overwritten
 *   workspace          device, >= the size above, 256-byte aligned
 * Constraints: those of nsa_compress; l * N2 * 4 bytes at most 4 MiB
 * (NSA_ERR_UNSUPPORTED beyond).  Deterministic: dw is summed in partial sums
 * over runs of consecutive compressed rows (in the workspace), then over the
 * runs in run order.  Three launches for dk / dv, dw partials and their sum.
 */
nsa_status_t nsa_compress_backward(
    const void* k, const void* v, const void* w, const float* dkcmp, const float* dvcmp, int l, int d,
    const int32_t* cu_seqlens, int batch, int n2, int d1, int d2, nsa_dtype_t dtype,
    float* dk, float* dv, float* dw, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream` and reads the device error word of `workspace`
 * (written by the last nsa_compress_attention, nsa_select_attention or
 * nsa_compress_attention_backward that used it).  Returns NSA_OK,
 * NSA_ERR_TIMEOUT when a device-side wait gave up, or NSA_ERR_CUDA.
 */
nsa_status_t nsa_workspace_status(const void* workspace, void* stream);

/*
 * Device-side error word of the compress kernel on the current device
 * (0 = none).  Synchronises `stream`.  NSA_ERR_TIMEOUT when a wait gave up,
 * NSA_ERR_INVALID_ARG when nsa_compress_paged met a block-table entry outside
 * its pool.
 */
nsa_status_t nsa_compress_status(void* stream);

/*
 * Same computation, outputs and argument rules as nsa_compress_attention,
 * for callers that cannot allocate device memory: for example an application
 * that has already claimed almost all of the GPU's memory for its own pools,
 * a plugin that is handed only the tensors it works on, or a path where an
 * allocation call is not permitted.  The source pages have no counterpart of
 * this call.
 *   - No workspace argument: the library uses its own fixed scratch array of
 *     16 MiB per device (a static device array that every GPU which loads
 *     the library keeps until the process exits).  When the workspace that
 *     nsa_compress_attention_workspace_size reports exceeds 16 MiB, the call
 *     runs on fewer persistent CTAs (each CTA needs its own importance
 *     scratch), then with one M-tile per work item, until it fits: same
 *     results, lower throughput.  Arguments for which even one CTA's scratch
 *     exceeds 16 MiB are rejected with NSA_ERR_WORKSPACE before anything is
 *     enqueued.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *     Under CUDA's lazy module loading (the default since CUDA 12.2) the
 *     array's 16 MiB are committed on a device when the library's module is
 *     first loaded there, which is this first call: make it before the
 *     application claims the rest of the device's memory for its own pools.
 *     The looked-up address is kept per device ordinal; a cudaDeviceReset
 *     invalidates it, so do not call this entry point after one.
 *   - All calls on a device share the one array, which keeps the contents of
 *     the last call; each call rewrites the parts that must start at zero.
 *     Calls whose work can overlap on the GPU (different streams without
 *     ordering between them) race on the array and must not be issued.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *     routine.
 */
nsa_status_t nsa_compress_attention_noalloc(
    const void* q, const void* kcmp, const void* vcmp, float scale, int head_num,
    int l, int d, int lp, int count,
    const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
    int batch, int n2, int d1, int d2, nsa_dtype_t dtype,
    void* attention_out, int32_t* topk_indices, float* softmax_max, float* softmax_sum,
    void* stream);

/*
 * Device error word of the last nsa_compress_attention_noalloc on the
 * current device (the counterpart of nsa_workspace_status for the fixed
 * scratch array, which the caller has no pointer to).  Synchronises `stream`
 * first.  Returns NSA_OK, NSA_ERR_TIMEOUT when a device-side wait of that
 * call gave up (its outputs are then not valid), or NSA_ERR_CUDA.
 */
nsa_status_t nsa_noalloc_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NSA_B200_H */
