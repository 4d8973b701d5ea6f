// nsa_internal.h -- structures shared by the host launcher (nsa_api.cu) and
// the kernels.  Not part of the public C ABI.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace nsa {

// ------------------------------------------------------------ compress
constexpr int kCompressStages = 2;        // shared-memory ring depth
constexpr int kCompressMaxThreads = 512;  // one thread per 16-byte column vector
constexpr int kCompressMaxSeq = 96;       // sequences per launch (kernel-parameter space)

// Device error word value: a block-table entry outside the page pool (the
// store it addressed was skipped).
constexpr int kErrBadPage = 0x200;
// Debug builds (NSA_DEBUG): a computed global index outside its tensor; the
// access was skipped.  kErrBounds + the id of the checking site.
constexpr int kErrBounds = 0x300;

#ifdef __CUDACC__
// Debug-build bounds check of a computed global index: false (and the first
// such site recorded in *err) when `ok` fails; release builds compile it away.
__device__ __forceinline__ bool nsa_index_ok(bool ok, int* err, int site) {
#ifdef NSA_DEBUG
    if (!ok && err != nullptr) atomicCAS(err, 0, kErrBounds + site);
    return ok;
#else
    (void)err;
    (void)site;
    (void)ok;
    return true;
#endif
}
#endif

struct CompressSeq {
    int raw_start;   // first raw row of the sequence (T2 index)
    int cmp_start;   // first compressed row (Tc index)
    int ncmp;        // compressed blocks of the sequence
    int first;       // first block computed (blocks first .. ncmp-1)
    int seq;         // sequence index (block-table row)
    int nchunks;     // CTAs given to the sequence
    int chunk_end;   // inclusive prefix of nchunks over the launch's sequences
};

struct CompressParams {
    const void* k;
    const void* v;
    const void* w;
    void* kcmp;
    void* vcmp;
    int l, d, n2, d1, d2;
    int dtype;            // 0 bf16, 1 fp16
    int chunk;            // output blocks per CTA
    int rows_per_stage;   // raw rows per bulk copy
    // paged output: block i of sequence b goes to row i % page_rows of pool page
    // block_table[b * bt_stride + i / page_rows] (null: contiguous, row cmp_start + i)
    const int32_t* block_table;
    int bt_stride, page_rows, num_pages;
    long long tc_rows;    // rows of the contiguous outputs (debug bounds checks)
    int nseq;
    CompressSeq seq[kCompressMaxSeq];
};

cudaError_t launch_compress(const CompressParams& p, dim3 grid, int threads, size_t smem,
                            cudaStream_t st);
cudaError_t read_compress_error(int* out, cudaStream_t st);

// ----------------------------------------------------------- attention
// One pass of online softmax per M-tile.  Warp roles (512 threads, four
// warpgroups): warps 0-3 softmax of pipeline 0, warps 4-7 softmax of
// pipeline 1 (idle when the launch runs one pipeline), warps 8-11 epilogue
// (output, group sums, top-k), warp 12 TMA producer, warp 13 MMA issuer,
// warps 14-15 idle.  Launched at 128 registers per thread (512 x 128 =
// 65536); setmaxnreg then moves registers to the softmax warpgroups.
constexpr int kAttnThreads = 512;
constexpr int kRegsSoftmax = 176;
constexpr int kRegsEpilogue = 96;
constexpr int kRegsCtl = 64;
static_assert((2 * kRegsSoftmax + kRegsEpilogue + kRegsCtl) * 128 <= kAttnThreads * 128,
              "register split exceeds the launch allocation");
constexpr int kRows = 128;          // M of one tile: (tokens x heads of one KV group)
constexpr float kRescaleLog2 = 8.f; // a row's reference maximum moves only when a
                                    // chunk's maximum exceeds it by more than this

// One work item: up to npipe x (128/G) consecutive query tokens of one
// sequence x the G heads of one KV group.  Pipeline p takes the tokens
// [p*TT, (p+1)*TT) of the item (TT = 128/G), one 128-row M-tile each; both
// read the same K/V tiles.
struct AttnTile {
    int q_row0;     // first query row (T1 index)
    int ntok;       // tokens in the item (<= npipe * TT)
    int group;      // KV head g
    int cmp_row0;   // first compressed row of the sequence (Tc index)
    int n_cmp;      // compressed blocks of the sequence
    int n_sel;      // selection blocks of the sequence
    int t0;         // position of the first token (query offset applied)
    int nkv;        // KV tiles to visit
    int tloc0;      // query index of the first token inside its sequence (mask rows)
    int seq;        // sequence index (block-table row)
};

struct AttnParams {
    const AttnTile* tiles;
    int num_tiles;
    int* err;               // device error word (workspace)
    // paged compressed K/V: when block_table is set, sequence b's compressed rows
    // j*page_rows .. live in pool page block_table[b * bt_stride + j] (the tensor
    // maps cover the pools, pool_rows rows, with boxes of page_rows rows)
    const int32_t* block_table;
    int bt_stride, page_rows, pool_rows;
    long long rows_q;       // rows of q and of the outputs (debug bounds checks)
    // two passes: exact row maxima and sums first, then normalised P, whose band
    // values the softmax sums over a token's G heads on chip (one score row per
    // token in the scratch); for 128-block KV tiles and G a power of two <= 32
    int two_pass;
    // per-CTA scratch for the per-head importance values: for each pipeline,
    // two slots (consecutive items alternate) of `region` floats each.  A slot
    // holds the banded values chunk-major, [chunk][row 0..127][anchor of the
    // chunk] (capj floats), then the reference maximum each chunk was written
    // against, row-major, [row][chunk] with row stride capc.
    float* band;
    int capj, capc, region;
    float* score_gmem;      // per-warp score rows when they do not fit on chip
    int score_cap;          // floats per score row
    int score_in_smem;
    void* out;
    int32_t* topk;
    float* smax;
    float* ssum;
    int dtype;              // 0 bf16, 1 fp16
    int n1, n2, d1, d2, G, tok_per_tile;
    int l, d, lp, count, a, b;
    float scale_log2;       // scale * log2(e)
    int nkv_cols;           // compressed blocks per KV tile
    int nslot;              // K/V ring depth
    int nqbuf;              // Q buffers (each holds npipe M-tiles of Q)
    int npipe;              // M-tiles per item (1 or 2)
    int nsb;                // score buffers per pipeline in tensor memory
    int tm_s[2], tm_o[2];   // tensor-memory columns: score buffer 0 and O of each pipeline
    // shared-memory layout (byte offsets from a 1024-aligned base)
    int off_q, q_bytes, off_ring, slot_bytes, off_rowstat, off_score, off_bar, smem_bytes;
    // optional masks (null = none): bool bytes (S1, row stride), one matrix for
    // every sequence and head, row = query index inside the sequence
    const uint32_t* am_bits;   // atten_mask bit-packed, am_words words per mask row (step 1)
    int am_words;
    const uint32_t* tm_bits;   // topk_mask bit-packed, tm_words words per mask row (step 6)
    int tm_words;
};

// byte mask (rows x s2) -> bit rows of `words` words, columns >= ncols cleared
cudaError_t launch_pack_mask(const uint8_t* src, long long s2, int ncols, int rows, int words, uint32_t* dst,
                             cudaStream_t st);
cudaError_t launch_attention(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, int grid, cudaStream_t st);
int attention_kv_cols(int a);     // compressed blocks per KV tile for band factor a
int attention_chunk_cols(int a);  // score columns per softmax chunk for band factor a

// ------------------------------------------------------------ backward
// Gradients of steps 1-3 (attention_out) with respect to q, kcmp and vcmp,
// and of the compression with respect to the raw K/V rows and w.
namespace bwd {
constexpr int kThreads = 160;    // warps 0-3 softmax (TMEM lane quadrants), warp 4 TMA + MMA
constexpr int kThreadsDq = 288;  // dQ: warps 0-3 and 5-8 softmax (two per lane quadrant), warp 4 TMA + MMA
constexpr int kKV = 128;         // compressed blocks per KV tile

// dQ: one query M-tile (TT tokens x G heads of one group) over its KV tiles
struct QItem {
    int q_row0, ntok, group, cmp_row0, n_cmp, t0, nkv;
};
// dK/dV: one KV tile of one group over a run of the query M-tiles that see
// it; the run's partial sums go to partial slot `slot`
struct KVItem {
    int cmp_row0;   // first compressed row of the sequence
    int kt;         // KV tile index inside the sequence
    int n_cmp;      // compressed blocks of the sequence
    int group;
    int q_row0;     // first query row of the run
    int q_end;      // end of the run's query rows
    int t0;         // position of query row q_row0 (query offset applied)
    int slot;       // partial slot: 128 rows x (D2 + D1) fp32
};
// One KV tile's partial slots [slot0, slot0 + nslots), summed in order
struct KVTile {
    int cmp_row0, kt, n_cmp, group, slot0, nslots;
};

struct Params {
    const QItem* qitems;
    int n_qitems;
    const KVItem* kvitems;
    int n_kvitems;
    int* err;
    const float2* rowinfo;   // (T1, N1): log2 normaliser m*log2e + log2 L (inf: row sees nothing), delta
    float* dq;               // (T1, N1, D1) fp32
    float* part;             // partial slots of dK/dV: [slot][128][D2 | D1] fp32
    long long rows_q, rows_c, n_slots;   // extents for debug bounds checks
    int mode;                // dK/dV kernel: bit 0 dV, bit 1 dK
    int col_dk;              // tensor-memory column of the dK accumulator
    int nsb;                 // dK/dV kernel: score buffers (2 when the accumulators end by column 256)
    int dtype, n1, n2, d1, d2, G, tok_per_tile, l, d;
    float scale, scale_log2;
    // shared memory (byte offsets from a 1024-aligned base) of the launched kernel: stage 0 of
    // each operand; the ring's stages (Q/dO for dK/dV, K/V for dQ) are stage_bytes apart
    int off_q, off_do, off_k, off_v, off_row, off_bar, smem_bytes;
    int nst, stage_bytes;
};

cudaError_t launch_prep(const void* out, const void* dout, const float* smax, const float* ssum, float2* rowinfo,
                        long long rows, int d2, int dtype, cudaStream_t st);
cudaError_t launch_dq(const Params& p, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                      const CUtensorMap& tv, cudaStream_t st);
cudaError_t launch_dkdv(const Params& p, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                        const CUtensorMap& tv, cudaStream_t st);
// dkcmp / dvcmp rows of every KV tile from its partial slots (dK scaled)
cudaError_t launch_reduce(const KVTile* tiles, int ntiles, const float* part, float* dkcmp, float* dvcmp, int n2,
                          int d1, int d2, float scale, long long rows_c, int* err, cudaStream_t st);

constexpr int kRowsPerCta = 32;   // raw rows per CTA of the compression transpose
struct CompressBwdSeq {
    int raw_start, raw_len, cmp_start, n_cmp;
    int blk_end;                  // inclusive prefix of the sequences' row blocks in this launch
};
struct CompressBwdParams {
    const void* k;
    const void* v;
    const void* w;
    const float* dkcmp;
    const float* dvcmp;
    float* dk;
    float* dv;
    float* dw;
    const int* cmp_raw;           // per compressed row: its first raw row (T2 index)
    float* dw_part;               // dw partial sums, [run][l][n2]
    int dw_run;                   // compressed rows per dw run
    long long tc;
    long long t2;                 // raw rows (debug bounds checks)
    int l, d, n2, d1, d2, dtype;
    int nseq;
    CompressBwdSeq seq[kCompressMaxSeq];
};
// dk, dv for the launch's sequences (one call per batch of sequences)
cudaError_t launch_compress_bwd_dx(const CompressBwdParams& p, int blocks, cudaStream_t st);
// dw over every compressed row: partial sums per run of p.dw_run rows, then their
// sum in run order (two launches)
int compress_dw_heads_per_cta(int d, int n2);   // heads of one dw partial-sum CTA
cudaError_t launch_compress_bwd_dw(const CompressBwdParams& p, int nruns, cudaStream_t st);
}  // namespace bwd

// ------------------------------------------------ selection attention
// Attention over the raw K/V blocks of l' tokens that the compressed branch's
// top-k lists per (query row, KV group).  Same warp roles and register split
// as the compressed-attention kernel.
namespace sel {
constexpr int kThreads = 192;      // warps 0-3 softmax + output, 4 TMA, 5 MMA
constexpr int kThreadsSplit = 320; // and warps 6-9 softmax when a KV tile splits in two halves
constexpr int kXchgBytes = 3072;   // per-row maxima and sums exchanged by the two halves
constexpr int kMaxSBuf = 8;        // score buffers in tensor memory
constexpr int kBarBytes = 512;     // mbarriers, tensor-memory address, abort flag
constexpr int kPlanThreads = 256;
// listed blocks of lp keys placed side by side in one KV tile: 128 keys when
// lp divides 128, else one block per tile
constexpr int blocks_per_tile(int lp) { return (128 % lp == 0) ? 128 / lp : 1; }
// whether the attention kernel for l' = lp splits a KV tile between two softmax warps per
// lane quadrant: tiles of several listed blocks whose halves are whole tensor-memory pieces
// (measured on B200: 16K and varlen workloads (l' = 64) 6-7 % faster; with one 128-key block
// per tile (l' = 128) 3 % slower, the per-tile exchange of row maxima costing more than the
// halved arithmetic saves)
constexpr bool attn_split(int lp) { return blocks_per_tile(lp) >= 2 && (blocks_per_tile(lp) * lp) % 32 == 0; }
constexpr int attn_threads(int lp) { return attn_split(lp) ? kThreadsSplit : kThreads; }

// One M-tile: up to 128/G consecutive query tokens of one sequence x the G
// heads of one KV group.
struct Tile {
    int q_row0;     // first query row (T1 index)
    int ntok;       // tokens in the tile
    int group;      // KV head g
    int kv_row0;    // first raw K/V row of the sequence (T2 index)
    int s_kv;       // K/V length of the sequence
    int t0;         // key position of the first token (bottom-right alignment)
    int n_blk;      // selection blocks of the sequence: ceil(s_kv / l')
    int pad;
};

struct Params {
    const Tile* tiles;
    int num_tiles;
    int* err;                   // device error word (workspace)
    long long rows_q;           // rows of q and of the outputs (debug bounds checks)
    const int32_t* topk;        // (T1, N2, count) block lists
    int count;
    int* list_n;                // per tile: blocks in the union of its tokens' lists
    int32_t* list_blk;          // per tile: cap block indices, ascending
    uint32_t* list_mask;        // per tile: cap x 4 words, bit tau = token tau listed the block
    int cap;                    // list capacity per tile
    void* out;
    float* lse;
    int dtype;                  // 0 bf16, 1 fp16
    int n1, n2, d1, d2, G, tok_per_tile, lp;
    float scale_log2;           // scale * log2(e)
    int nslot, nqbuf, nsbuf;    // K/V ring depth, Q buffers, S buffers
    int tm_o;                   // tensor-memory column of O (d2 columns)
    int tm_s, s_stride;         // column of score buffer 0, columns between buffers
    // shared-memory layout (byte offsets from a 1024-aligned base)
    int off_q, q_bytes, off_ring, slot_bytes, off_bar, off_x, smem_bytes;
};

cudaError_t launch_plan(const Params& p, int max_words, cudaStream_t st);
cudaError_t launch_attention(const Params& p, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, int grid, cudaStream_t st);
}  // namespace sel

}  // namespace nsa
