// nsa_api.cu -- the C ABI: argument validation, work decomposition, tensor
// maps and launches.  Validation returns a status before anything is enqueued
// ("aclnnNsaCompress": the first phase checks the parameters and returns a
// status code); the launches are asynchronous on the caller's stream.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/nsa.h"
#include "nsa_internal.h"

using namespace nsa;

namespace {

constexpr size_t kWsHeader = 256;     // error word + padding
constexpr int kMaxGrid = 160;         // persistent CTAs sized for one CTA per SM (148 on B200)
constexpr int kSmemLimit = 232448;    // dynamic shared memory per block on sm_100

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

nsa_status_t check_prefix(const int32_t* cu, int batch) {
    if (cu == nullptr || batch < 1) return NSA_ERR_INVALID_ARG;
    int32_t prev = 0;
    for (int b = 0; b < batch; ++b) {
        if (cu[b] < prev) return NSA_ERR_INVALID_ARG;   // prefix sums never decrease
        prev = cu[b];
    }
    return NSA_OK;
}

// Status of a device error word: a timed-out wait, a block-table entry outside
// its pool, or (debug builds) a computed index outside its tensor.
nsa_status_t error_status(int err) {
    if (err == 0) return NSA_OK;
    if (err == kErrBadPage || (err >= kErrBounds && err < kErrBounds + 0x100)) return NSA_ERR_INVALID_ARG;
    return NSA_ERR_TIMEOUT;
}

int64_t ncmp_of(int64_t S, int l, int d) {
    // aclnnNsaCompress Formula: blocks i = 0 .. floor((S-l)/d); none when S < l
    return S < l ? 0 : (S - l) / d + 1;
}

inline int nvis_host(int64_t t, int l, int d, int n_cmp) {
    if (t < l - 1) return 0;
    return (int)std::min<int64_t>(n_cmp, (t - l + 1) / d + 1);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3D map over a TND tensor (D contiguous, then N, then T), 64-element boxes
// along D with 128-byte swizzle.
bool encode_tnd(CUtensorMap* map, const void* base, int dtype, int D, int N, int64_t T, int box_n,
                int box_t) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)std::max<int64_t>(T, 1)};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * N * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)box_n, (cuuint32_t)box_t};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, dtype == 0 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------------
// attention plan: everything derived from the host arguments
// ------------------------------------------------------------------------
struct AttnPlan {
    int G = 0, TT = 0, a = 0, b = 0, nkv_cols = 0, chunk = 0, npipe = 1, nsb = 2;
    int64_t max_sq = 0;   // queries of the longest sequence
    std::vector<AttnTile> tiles;
    int score_cap = 4;
    int grid = 0, max_nkv = 0, capj = 4, capc = 4, region = 64;
    bool score_in_smem = true;
    int nslot = 0, nqbuf = 1, tm_s[2] = {0, 0}, tm_o[2] = {0, 0};
    int off_q = 0, q_bytes = 0, off_ring = 0, slot_bytes = 0, off_rowstat = 0, off_score = 0, off_bar = 0,
        smem_bytes = 0;
    size_t ws_tiles = 0, ws_score = 0, ws_band = 0, ws_total = 0;
    size_t ws_fixed = 0, ws_per_cta = 0;   // ws_total = ws_fixed + grid * ws_per_cta
};

nsa_status_t validate_attention(int head_num, int n2, int d1, int d2, int l, int d, int lp, int count,
                                const int32_t* cu_q, const int32_t* cu_cmp, const int32_t* cu_sel,
                                int batch) {
    // note list of mindspore.ops.nsa_compress_attention
    if (l % 16 || d % 16 || lp % 16) return NSA_ERR_INVALID_ARG;
    if (l < 16 || l > 128 || d < 16 || d > 64 || lp < 16 || lp > 128) return NSA_ERR_INVALID_ARG;
    if (l < d || lp < l || lp % d) return NSA_ERR_INVALID_ARG;
    if (count < 1 || count > 32) return NSA_ERR_INVALID_ARG;
    if (d1 < 16 || d2 < 16 || d1 % 16 || d2 % 16 || d1 < d2) return NSA_ERR_INVALID_ARG;
    if (n2 < 1 || head_num < n2 || head_num % n2) return NSA_ERR_INVALID_ARG;
    nsa_status_t s;
    if ((s = check_prefix(cu_q, batch)) != NSA_OK) return s;
    if ((s = check_prefix(cu_cmp, batch)) != NSA_OK) return s;
    if ((s = check_prefix(cu_sel, batch)) != NSA_OK) return s;
    // beyond the pages' constraints: what this build runs
    if (l % d) return NSA_ERR_UNSUPPORTED;          // l/d must be an integer in step 4
    if (d1 > 256 || d2 > 256) return NSA_ERR_UNSUPPORTED;
    if (head_num / n2 > kRows) return NSA_ERR_UNSUPPORTED;
    return NSA_OK;
}

// Work items of npipe x TT tokens; grid_cap bounds the persistent grid (and
// with it the per-CTA scratch of the workspace); npipe_max = 1 forces one
// M-tile per item.
nsa_status_t plan_attention(int head_num, int n2, int d1, int d2, int l, int d, int lp, int count,
                            const int32_t* cu_q, const int32_t* cu_cmp, const int32_t* cu_sel, int batch,
                            bool build_tiles, AttnPlan& pl, int grid_cap = kMaxGrid, int npipe_max = 2,
                            int group_begin = 0, int group_count = -1) {
    nsa_status_t s = validate_attention(head_num, n2, d1, d2, l, d, lp, count, cu_q, cu_cmp, cu_sel, batch);
    if (s != NSA_OK) return s;
    if (group_count < 0) group_count = n2 - group_begin;
    if (group_begin < 0 || group_count < 0 || group_begin + group_count > n2) return NSA_ERR_INVALID_ARG;
    const int g_end = group_begin + group_count;
    pl.G = head_num / n2;
    pl.TT = kRows / pl.G;
    pl.a = lp / d;
    pl.b = l / d;
    pl.nkv_cols = attention_kv_cols(pl.a);
    pl.chunk = attention_chunk_cols(pl.a);
    const int NKV = pl.nkv_cols;
    const int NCH = NKV / pl.chunk;
    const int NJ = NKV / pl.a;
    const int NJC = pl.chunk / pl.a;

    // score-row capacity (largest candidate count) and the longest KV walk
    int cap = 1, max_nkv = 0;
    int64_t max_sq = 0;
    {
        int32_t pq = 0, pc = 0, ps = 0;
        for (int bq = 0; bq < batch; ++bq) {
            const int64_t Sq = cu_q[bq] - pq;
            const int n_cmp = cu_cmp[bq] - pc;
            const int n_sel = cu_sel[bq] - ps;
            const int64_t off = n_cmp > 0 ? std::max<int64_t>(0, (int64_t)(n_cmp - 1) * d + l - Sq) : 0;
            max_sq = std::max(max_sq, Sq);
            if (Sq > 0) {
                const int64_t tlast = Sq - 1 + off;
                const int nv = nvis_host(tlast, l, d, n_cmp);
                if (nv > 0) cap = std::max<int64_t>(cap, std::min<int64_t>(n_sel, tlast / lp + 1));
                max_nkv = std::max(max_nkv, (nv + NKV - 1) / NKV);
            }
            pq = cu_q[bq];
            pc = cu_cmp[bq];
            ps = cu_sel[bq];
        }
    }
    pl.max_sq = max_sq;
    pl.score_cap = (cap + 3) & ~3;
    pl.max_nkv = max_nkv;
    // importance scratch of one slot: chunks of every KV tile plus the one past
    // the last (its first anchors still collect taps), 128 rows each
    const int nchk = max_nkv * NCH + 1;
    pl.capj = nchk * kRows * NJC;
    pl.capc = (nchk + 3) & ~3;
    pl.region = (pl.capj + kRows * pl.capc + 63) & ~63;

    // shared memory: Q buffers (npipe M-tiles each), K/V ring, row statistics,
    // per-warp score rows, mbarriers.  Tensor memory: with two pipelines one
    // score buffer and O each (O within 128 columns); with one, two score
    // buffers and O.
    const int nqc = (d1 + 63) / 64, nvc = (d2 + 63) / 64;
    const int score_bytes = 4 * pl.score_cap * 4;
    const int rowstat_bytes = (2 * 2 * 2 * kRows + 4 * kRows) * 4;   // row statistics + per-warp normalisers
    const int bar_bytes = 512;
    pl.slot_bytes = std::max(nqc, nvc) * NKV * 128;
    auto layout = [&](int np, int nq, int ns, bool in_smem) {
        int off = 0;
        pl.q_bytes = np * nqc * 16384;
        pl.off_q = off;
        off += nq * pl.q_bytes;
        pl.off_ring = off;
        off += ns * pl.slot_bytes;
        pl.off_rowstat = off;
        off += rowstat_bytes;
        pl.off_score = off;
        if (in_smem) off += (score_bytes + 127) & ~127;
        pl.off_bar = off;
        off += bar_bytes;
        pl.smem_bytes = off + 1024;   // slack for 1024-byte alignment of the base
        pl.npipe = np;
        pl.nqbuf = nq;
        pl.nslot = ns;
        pl.score_in_smem = in_smem;
        return pl.smem_bytes <= kSmemLimit;
    };
    // preference: a K/V ring of at least three slots, then two pipelines, a
    // deeper ring, a second Q buffer, on-chip score rows.  Measured on B200:
    // with D1 = 192 two pipelines leave two ring slots and run slower than one
    // pipeline with three (varlen workload 7.2 vs 6.6 ms)
    static const int kOrder[][2] = {{2, 4}, {2, 3}, {1, 4}, {1, 3}};
    static const int kOrder2[][2] = {{2, 2}, {1, 2}};
    bool fits = false;
    // a second pipeline needs a second M-tile of tokens: when every sequence's queries
    // fit one M-tile (decode, few queries), one pipeline with two score buffers
    const int np_hi = std::min(npipe_max, (d2 <= 128 && max_sq > pl.TT) ? 2 : 1);
    for (int np = np_hi; np >= 1 && !fits; --np)
        for (const auto& o : kOrder) {
            if ((fits = layout(np, o[0], o[1], true))) break;
            if ((fits = layout(np, o[0], o[1], false))) break;
        }
    for (int np = np_hi; np >= 1 && !fits; --np)
        for (const auto& o : kOrder2) {
            if ((fits = layout(np, o[0], o[1], true))) break;
            if ((fits = layout(np, o[0], o[1], false))) break;
        }
    if (!fits) return NSA_ERR_UNSUPPORTED;
    if (pl.npipe == 2) {
        pl.nsb = 1;
        pl.tm_s[0] = 0;
        pl.tm_s[1] = 128;
        pl.tm_o[0] = 256;
        pl.tm_o[1] = 384;
    } else {
        pl.nsb = 2;
        pl.tm_s[0] = pl.tm_s[1] = 0;
        pl.tm_o[0] = pl.tm_o[1] = 256;
        if (256 + d2 > 512) return NSA_ERR_UNSUPPORTED;
    }

    // items: (sequence, group, run of npipe * TT tokens)
    const int run = pl.npipe * pl.TT;
    int64_t ntiles = 0;
    {
        int32_t pq = 0;
        for (int bq = 0; bq < batch; ++bq) {
            const int64_t Sq = cu_q[bq] - pq;
            ntiles += ((Sq + run - 1) / run) * (int64_t)group_count;
            pq = cu_q[bq];
        }
    }
    if (ntiles > (int64_t)1 << 30) return NSA_ERR_UNSUPPORTED;
    pl.grid = (int)std::max<int64_t>(1, std::min<int64_t>(ntiles, std::max(1, grid_cap)));

    if (build_tiles) {
        pl.tiles.clear();
        pl.tiles.reserve((size_t)ntiles);
        int32_t pq = 0, pc = 0, ps = 0;
        for (int bq = 0; bq < batch; ++bq) {
            const int Sq = cu_q[bq] - pq;
            const int n_cmp = cu_cmp[bq] - pc;
            const int n_sel = cu_sel[bq] - ps;
            const int64_t off = n_cmp > 0 ? std::max<int64_t>(0, (int64_t)(n_cmp - 1) * d + l - Sq) : 0;
            for (int tok0 = 0; tok0 < Sq; tok0 += run) {
                AttnTile t;
                t.q_row0 = pq + tok0;
                t.ntok = std::min(run, Sq - tok0);
                t.cmp_row0 = pc;
                t.n_cmp = n_cmp;
                t.n_sel = n_sel;
                t.t0 = (int)(tok0 + off);
                t.tloc0 = (int)tok0;
                t.seq = bq;
                const int nv = nvis_host(t.t0 + t.ntok - 1, l, d, n_cmp);
                t.nkv = (nv + NKV - 1) / NKV;
                for (int g = group_begin; g < g_end; ++g) {
                    t.group = g;
                    pl.tiles.push_back(t);
                }
            }
            pq = cu_q[bq];
            pc = cu_cmp[bq];
            ps = cu_sel[bq];
        }
        // longest items first: with the round-robin hand-out of the persistent
        // grid this approximates longest-processing-time-first scheduling
        std::stable_sort(pl.tiles.begin(), pl.tiles.end(),
                         [](const AttnTile& x, const AttnTile& y) { return x.nkv > y.nkv; });
    }

    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    pl.ws_tiles = (size_t)ntiles * sizeof(AttnTile);
    const size_t score_per_cta = pl.score_in_smem ? 0 : (size_t)4 * pl.score_cap * 4;
    const size_t band_per_cta = (size_t)pl.npipe * 2 * (size_t)pl.region * 4;
    pl.ws_score = up((size_t)pl.grid * score_per_cta);
    pl.ws_band = up((size_t)pl.grid * band_per_cta);
    pl.ws_fixed = kWsHeader + up(pl.ws_tiles) + 512;
    pl.ws_per_cta = score_per_cta + band_per_cta;
    pl.ws_total = kWsHeader + up(pl.ws_tiles) + pl.ws_score + pl.ws_band;
    return NSA_OK;
}

// Bit-packed copies of the optional masks, placed after the attention
// workspace: max_q rows each; atten_mask rows cover every column a KV tile
// walk reads (plus a two-word window tail), topk_mask rows every candidate.
struct MaskPack {
    int64_t rows = 0, max_c = 0, max_s = 0;
    int am_words = 0, tm_words = 0;
    size_t am_bytes = 0, tm_bytes = 0;
};

MaskPack plan_masks(const AttnPlan& pl, const int32_t* cu_q, const int32_t* cu_cmp, const int32_t* cu_sel,
                    int batch, bool am, bool tm) {
    MaskPack m;
    for (int b = 0; b < batch; ++b) {
        m.rows = std::max<int64_t>(m.rows, cu_q[b] - (b ? cu_q[b - 1] : 0));
        m.max_c = std::max<int64_t>(m.max_c, cu_cmp[b] - (b ? cu_cmp[b - 1] : 0));
        m.max_s = std::max<int64_t>(m.max_s, cu_sel[b] - (b ? cu_sel[b - 1] : 0));
    }
    auto words = [](int64_t cols) { return (int)((((cols + 31) / 32 + 2) + 1) & ~int64_t(1)); };
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    if (am) {
        m.am_words = words((int64_t)pl.max_nkv * pl.nkv_cols);
        m.am_bytes = up((size_t)m.rows * m.am_words * 4);
    }
    if (tm) {
        m.tm_words = words(m.max_s);
        m.tm_bytes = up((size_t)m.rows * m.tm_words * 4);
    }
    return m;
}

// ------------------------------------------------------------------------
// selection-attention plan
// ------------------------------------------------------------------------
struct SelPlan {
    int G = 0, TT = 0, cap = 1, max_words = 1, grid = 0;
    std::vector<sel::Tile> tiles;
    int nslot = 0, nqbuf = 1, nsbuf = 2, tm_o = 0, tm_s = 0, s_stride = 0;
    int off_q = 0, q_bytes = 0, off_ring = 0, slot_bytes = 0, off_bar = 0, off_x = 0, smem_bytes = 0;
    size_t ws_tiles = 0, ws_n = 0, ws_blk = 0, ws_mask = 0, ws_total = 0;
};

nsa_status_t plan_select(int head_num, int n2, int d1, int d2, int lp, int count, const int32_t* cu_q,
                         const int32_t* cu_kv, int batch, bool build_tiles, SelPlan& pl) {
    // block shape of the index lists: l' (select_block_size of the compressed
    // branch) keys per block; tiles of 16-column multiples for the MMA
    if (lp % 16 || lp < 16 || lp > 128) return NSA_ERR_INVALID_ARG;
    if (count < 1 || count > 32) return NSA_ERR_INVALID_ARG;
    if (d1 < 16 || d2 < 16 || d1 % 16 || d2 % 16) return NSA_ERR_INVALID_ARG;
    if (n2 < 1 || head_num < n2 || head_num % n2) return NSA_ERR_INVALID_ARG;
    nsa_status_t s;
    if ((s = check_prefix(cu_q, batch)) != NSA_OK) return s;
    if ((s = check_prefix(cu_kv, batch)) != NSA_OK) return s;
    if (d1 > 256 || d2 > 256) return NSA_ERR_UNSUPPORTED;
    if (head_num / n2 > kRows) return NSA_ERR_UNSUPPORTED;
    pl.G = head_num / n2;
    pl.TT = kRows / pl.G;
    int64_t ntiles = 0, max_blk = 1;
    {
        int32_t pq = 0, pk = 0;
        for (int bq = 0; bq < batch; ++bq) {
            const int64_t Sq = cu_q[bq] - pq, Skv = cu_kv[bq] - pk;
            ntiles += ((Sq + pl.TT - 1) / pl.TT) * (int64_t)n2;
            max_blk = std::max<int64_t>(max_blk, (Skv + lp - 1) / lp);
            pq = cu_q[bq];
            pk = cu_kv[bq];
        }
    }
    if (ntiles > (int64_t)1 << 30) return NSA_ERR_UNSUPPORTED;
    // the planning kernel keeps a bit map and a prefix word per 32 blocks on chip
    pl.max_words = (int)((max_blk + 31) / 32);
    if ((int64_t)pl.max_words * 8 > 200 * 1024) return NSA_ERR_UNSUPPORTED;
    pl.cap = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)pl.TT * count, max_blk));

    // tensor memory: O (d2 columns), then up to kMaxSBuf score buffers of one
    // KV tile each (P is written over the first half of its buffer), all at
    // 32-column boundaries
    pl.tm_o = 0;
    pl.tm_s = (d2 + 31) & ~31;
    const int nkv_keys = sel::blocks_per_tile(lp) * lp;     // keys per KV tile
    pl.s_stride = (nkv_keys + 31) & ~31;
    pl.nsbuf = std::min(sel::kMaxSBuf, (512 - pl.tm_s) / pl.s_stride);
    if (pl.nsbuf < 2) return NSA_ERR_UNSUPPORTED;
    // shared memory: Q buffers and the K/V ring
    const int nqc = (d1 + 63) / 64, nvc = (d2 + 63) / 64;
    pl.q_bytes = nqc * 16384;
    pl.slot_bytes = std::max(nqc, nvc) * nkv_keys * 128;
    auto layout = [&](int nq, int ns) {
        int off = 0;
        pl.off_q = off;
        off += nq * pl.q_bytes;
        pl.off_ring = off;
        off += ns * pl.slot_bytes;
        pl.off_bar = off;
        off += sel::kBarBytes;
        pl.off_x = off;
        off += sel::kXchgBytes;
        pl.smem_bytes = off + 1024;   // slack for 1024-byte alignment of the base
        pl.nqbuf = nq;
        pl.nslot = ns;
        return pl.smem_bytes <= kSmemLimit;
    };
    static const int kOrder[][2] = {{2, 8}, {2, 6}, {2, 4}, {1, 4}, {2, 2}, {1, 2}};
    bool fits = false;
    for (const auto& o : kOrder)
        if ((fits = layout(o[0], o[1]))) break;
    if (!fits) return NSA_ERR_UNSUPPORTED;
    // the kernel takes all 512 tensor-memory columns: keep a second CTA off the SM
    pl.smem_bytes = std::max(pl.smem_bytes, 120 * 1024);
    pl.grid = (int)std::min<int64_t>(ntiles, kMaxGrid);

    if (build_tiles) {
        pl.tiles.clear();
        pl.tiles.reserve((size_t)ntiles);
        // KV group outermost: the CTAs run neighbouring tiles at the same
        // time, and these then read the blocks of one group's K/V, which
        // stays in L2 while they do
        for (int g = 0; g < n2; ++g) {
            int32_t pq = 0, pk = 0;
            for (int bq = 0; bq < batch; ++bq) {
                const int Sq = cu_q[bq] - pq, Skv = cu_kv[bq] - pk;
                for (int tok0 = 0; tok0 < Sq; tok0 += pl.TT) {
                    sel::Tile t;
                    t.q_row0 = pq + tok0;
                    t.ntok = std::min(pl.TT, Sq - tok0);
                    t.group = g;
                    t.kv_row0 = pk;
                    t.s_kv = Skv;
                    t.t0 = tok0 + (Skv - Sq);
                    t.n_blk = (Skv + lp - 1) / lp;
                    t.pad = 0;
                    pl.tiles.push_back(t);
                }
                pq = cu_q[bq];
                pk = cu_kv[bq];
            }
        }
    }
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    pl.ws_tiles = up((size_t)ntiles * sizeof(sel::Tile));
    pl.ws_n = up((size_t)ntiles * 4);
    pl.ws_blk = up((size_t)ntiles * pl.cap * 4);
    pl.ws_mask = up((size_t)ntiles * pl.cap * 16);
    pl.ws_total = kWsHeader + pl.ws_tiles + pl.ws_n + pl.ws_blk + pl.ws_mask;
    return NSA_OK;
}

// ------------------------------------------------------------------------
// backward plan: dQ items, dK/dV runs and their partial slots
// ------------------------------------------------------------------------
struct BwdPlan {
    int G = 0, TT = 0;
    std::vector<bwd::QItem> qitems;
    std::vector<bwd::KVItem> kvitems;
    std::vector<bwd::KVTile> kvtiles;
    int nslots = 0;
    bool one_pass = true;   // dV and dK in one tensor-memory allocation
    int nst = 1, stage_bytes = 0, off_row = 0, off_bar = 0, smem_bytes = 0;
    size_t off_qitems = 0, off_kvitems = 0, off_kvtiles = 0, off_rowinfo = 0, off_part = 0, ws_total = 0;
};

nsa_status_t plan_backward(int head_num, int n2, int d1, int d2, int l, int d, const int32_t* cu_q,
                           const int32_t* cu_cmp, int batch, bool build, BwdPlan& pl) {
    // the forward's constraints (note list of mindspore.ops.nsa_compress_attention)
    if (l % 16 || d % 16 || l < 16 || l > 128 || d < 16 || d > 64 || l < d) return NSA_ERR_INVALID_ARG;
    if (d1 < 16 || d2 < 16 || d1 % 16 || d2 % 16 || d1 < d2) return NSA_ERR_INVALID_ARG;
    if (n2 < 1 || head_num < n2 || head_num % n2) return NSA_ERR_INVALID_ARG;
    nsa_status_t s;
    if ((s = check_prefix(cu_q, batch)) != NSA_OK) return s;
    if ((s = check_prefix(cu_cmp, batch)) != NSA_OK) return s;
    // what the kernels hold: Q, dO, K, V tiles on chip together
    const int nqc = (d1 + 63) / 64, nvc = (d2 + 63) / 64;
    if (d1 > 256 || d2 > 256 || nqc + nvc > 6) return NSA_ERR_UNSUPPORTED;
    if (head_num / n2 > kRows) return NSA_ERR_UNSUPPORTED;
    pl.G = head_num / n2;
    pl.TT = kRows / pl.G;
    pl.one_pass = d2 <= 128;
    const int TT = pl.TT, KV = bwd::kKV;

    // shared memory (one CTA per SM: the kernels take all 512 tensor-memory columns): the
    // fixed operands (Q/dO of a dQ item, K/V of a dK/dV tile), then one or two stages of the
    // streamed ones, the rows' statistics (two M-tile buffers) and the barriers
    pl.stage_bytes = (nqc + nvc) * 16384;
    auto fits = [&](int nst) {
        pl.nst = nst;
        pl.off_row = (1 + nst) * pl.stage_bytes;
        pl.off_bar = (pl.off_row + 2 * kRows * 12 + 127) & ~127;
        pl.smem_bytes = std::max(pl.off_bar + 128 + 1024, 116 * 1024);
        return pl.smem_bytes <= kSmemLimit;
    };
    if (!fits(2) && !fits(1)) return NSA_ERR_UNSUPPORTED;

    // total dK/dV work in M-tile steps, to size the runs: about four runs per SM
    auto first_row = [&](int kt, int64_t off_b) { return (int64_t)kt * KV * d + l - 1 - off_b; };
    int64_t steps = 0, nq = 0;
    {
        int32_t pq = 0, pc = 0;
        for (int b = 0; b < batch; ++b) {
            const int64_t Sq = cu_q[b] - pq;
            const int n_cmp = cu_cmp[b] - pc;
            const int64_t off_b = n_cmp > 0 ? std::max<int64_t>(0, (int64_t)(n_cmp - 1) * d + l - Sq) : 0;
            nq += (Sq + TT - 1) / TT;
            for (int kt = 0; kt * KV < n_cmp; ++kt) {
                const int64_t rows = Sq - std::max<int64_t>(0, first_row(kt, off_b));
                if (rows > 0) steps += (rows + TT - 1) / TT;
            }
            pq = cu_q[b];
            pc = cu_cmp[b];
        }
    }
    steps *= n2;
    nq *= n2;
    if (nq > ((int64_t)1 << 30)) return NSA_ERR_UNSUPPORTED;
    const int64_t run = std::max<int64_t>(8, (steps + 4 * kMaxGrid - 1) / (4 * kMaxGrid));   // M-tiles per run

    pl.qitems.clear();
    pl.kvitems.clear();
    pl.kvtiles.clear();
    pl.nslots = 0;
    int64_t nkvitems = 0, nkvtiles = 0, nslots = 0;
    {
        int32_t pq = 0, pc = 0;
        for (int b = 0; b < batch; ++b) {
            const int Sq = cu_q[b] - pq;
            const int n_cmp = cu_cmp[b] - pc;
            const int64_t off_b = n_cmp > 0 ? std::max<int64_t>(0, (int64_t)(n_cmp - 1) * d + l - Sq) : 0;
            for (int g = 0; g < n2; ++g) {
                if (build)
                    for (int tok0 = 0; tok0 < Sq; tok0 += TT) {
                        bwd::QItem it;
                        it.q_row0 = pq + tok0;
                        it.ntok = std::min(TT, Sq - tok0);
                        it.group = g;
                        it.cmp_row0 = pc;
                        it.n_cmp = n_cmp;
                        it.t0 = (int)(tok0 + off_b);
                        const int nv = nvis_host(it.t0 + it.ntok - 1, l, d, n_cmp);
                        it.nkv = (nv + KV - 1) / KV;
                        pl.qitems.push_back(it);
                    }
                for (int kt = 0; kt * KV < n_cmp; ++kt) {
                    const int64_t tl0 = std::max<int64_t>(0, first_row(kt, off_b));
                    const int64_t rows = std::max<int64_t>(0, Sq - tl0);
                    const int64_t nmt = (rows + TT - 1) / TT;
                    const int64_t nrun = (nmt + run - 1) / run;
                    if (build) {
                        bwd::KVTile t{pc, kt, n_cmp, g, (int)nslots, (int)nrun};
                        pl.kvtiles.push_back(t);
                        for (int64_t r = 0; r < nrun; ++r) {
                            bwd::KVItem it;
                            it.cmp_row0 = pc;
                            it.kt = kt;
                            it.n_cmp = n_cmp;
                            it.group = g;
                            it.q_row0 = (int)(pq + tl0 + r * run * TT);
                            it.q_end = (int)std::min<int64_t>(pq + Sq, it.q_row0 + run * TT);
                            it.t0 = (int)(tl0 + r * run * TT + off_b);
                            it.slot = (int)(nslots + r);
                            pl.kvitems.push_back(it);
                        }
                    }
                    nslots += nrun;
                    nkvitems += nrun;
                    ++nkvtiles;
                }
            }
            pq = cu_q[b];
            pc = cu_cmp[b];
        }
    }
    if (nslots > ((int64_t)1 << 24)) return NSA_ERR_UNSUPPORTED;
    pl.nslots = (int)nslots;
    if (build) {
        // longest first (the hardware hands CTAs out roughly in index order)
        std::stable_sort(pl.qitems.begin(), pl.qitems.end(),
                         [](const bwd::QItem& x, const bwd::QItem& y) { return x.nkv > y.nkv; });
        std::stable_sort(pl.kvitems.begin(), pl.kvitems.end(), [](const bwd::KVItem& x, const bwd::KVItem& y) {
            return x.q_end - x.q_row0 > y.q_end - y.q_row0;
        });
    }
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const int64_t t1 = cu_q[batch - 1];
    pl.off_qitems = kWsHeader;
    pl.off_kvitems = pl.off_qitems + up((size_t)nq * sizeof(bwd::QItem));
    pl.off_kvtiles = pl.off_kvitems + up((size_t)nkvitems * sizeof(bwd::KVItem));
    pl.off_rowinfo = pl.off_kvtiles + up((size_t)nkvtiles * sizeof(bwd::KVTile));
    pl.off_part = pl.off_rowinfo + up((size_t)t1 * head_num * sizeof(float2));
    pl.ws_total = pl.off_part + up((size_t)nslots * bwd::kKV * (d1 + d2) * sizeof(float));
    return NSA_OK;
}

}  // namespace

extern "C" {

const char* nsa_status_string(nsa_status_t s) {
    switch (s) {
        case NSA_OK: return "NSA_OK";
        case NSA_ERR_INVALID_ARG: return "NSA_ERR_INVALID_ARG";
        case NSA_ERR_UNSUPPORTED: return "NSA_ERR_UNSUPPORTED";
        case NSA_ERR_WORKSPACE: return "NSA_ERR_WORKSPACE";
        case NSA_ERR_CUDA: return "NSA_ERR_CUDA";
        case NSA_ERR_TIMEOUT: return "NSA_ERR_TIMEOUT";
    }
    return "NSA_ERR_UNKNOWN";
}

nsa_status_t nsa_compress_out_len(const int32_t* cu_seqlens, int batch, int l, int d, int32_t* cu_cmp_out,
                                  int64_t* total_out) {
    if (cu_cmp_out == nullptr || l < 1 || d < 1) return NSA_ERR_INVALID_ARG;
    nsa_status_t s = check_prefix(cu_seqlens, batch);
    if (s != NSA_OK) return s;
    int64_t tot = 0;
    int32_t prev = 0;
    for (int b = 0; b < batch; ++b) {
        tot += ncmp_of((int64_t)cu_seqlens[b] - prev, l, d);
        prev = cu_seqlens[b];
        if (tot > INT32_MAX) return NSA_ERR_INVALID_ARG;
        cu_cmp_out[b] = (int32_t)tot;
    }
    if (total_out) *total_out = tot;
    return NSA_OK;
}

}  // extern "C"

// Compression of blocks first_block[b] .. n_cmp_b - 1 of every sequence (all
// of them when first_block is null), into contiguous rows or, with a block
// table, into pages.
static nsa_status_t compress_impl(const void* k, const void* v, const void* w, int l, int d,
                                  const int32_t* cu_seqlens, int batch, int n2, int d1, int d2, nsa_dtype_t dtype,
                                  void* kcmp, void* vcmp, void* stream, const int32_t* first_block = nullptr,
                                  const int32_t* block_table = nullptr, int bt_stride = 0, int page_rows = 0,
                                  int64_t num_pages = 0) {
    // constraint lists of aclnnNsaCompress and mindspore.ops.nsa_compress_attention
    if (dtype != NSA_BF16 && dtype != NSA_FP16) return NSA_ERR_INVALID_ARG;
    if (k == nullptr || w == nullptr || kcmp == nullptr) return NSA_ERR_INVALID_ARG;
    if ((v == nullptr) != (vcmp == nullptr)) return NSA_ERR_INVALID_ARG;
    if (l % 16 || d % 16 || d < 16 || l < d || l > 128) return NSA_ERR_INVALID_ARG;
    if (n2 < 1 || d1 < 16 || d1 % 16 || d1 > 256) return NSA_ERR_INVALID_ARG;
    if (v && (d2 < 16 || d2 % 16 || d2 > 256)) return NSA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(kcmp) || (v && (!aligned16(v) || !aligned16(vcmp))))
        return NSA_ERR_INVALID_ARG;
    nsa_status_t s = check_prefix(cu_seqlens, batch);
    if (s != NSA_OK) return s;
    const int dmax = v ? std::max(d1, d2) : d1;
    const int64_t rowelems = (int64_t)n2 * dmax;
    if (rowelems / 8 > kCompressMaxThreads) return NSA_ERR_UNSUPPORTED;
    if ((int64_t)cu_seqlens[batch - 1] * rowelems > ((int64_t)1 << 40)) return NSA_ERR_UNSUPPORTED;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return NSA_ERR_CUDA;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);

    // sizes of the per-CTA ring and the output run of one CTA
    const int rowbytes = (int)(rowelems * 2);
    // rows per bulk copy: about 8 KB, a multiple of 4 (the kernel steps 4 rows at a time).
    // Measured on B200 against 16 KB and 32 KB stages and 3-8 deep rings, and, once
    // neighbouring runs shared their overlap rows through L2, against 3, 4 and 6 deep
    // rings of 8 KB: 8 KB x 2 gives the smallest CTAs (eight per SM, the register limit)
    // and the highest read rate (262144 tokens: 219 us against 229 / 234 / 261 us).
    int rs = std::max(4, (8192 / rowbytes) & ~3);
    const int stage_bytes = rs * rowbytes;
    const int wbytes = ((l * n2 * 4) + 127) & ~127;
    const size_t smem = (size_t)wbytes + 128 + (size_t)kCompressStages * stage_bytes;
    if (smem > (size_t)kSmemLimit) return NSA_ERR_UNSUPPORTED;
    const int occ = std::max(1, std::min(8, (int)(228 * 1024 / (smem + 1024))));
    int64_t total_out = 0;
    {
        int32_t prev = 0;
        for (int b = 0; b < batch; ++b) {
            const int64_t nc = ncmp_of((int64_t)cu_seqlens[b] - prev, l, d);
            const int64_t f = first_block ? first_block[b] : 0;
            if (f < 0 || f > nc) return NSA_ERR_INVALID_ARG;
            if (block_table && (nc + page_rows - 1) / page_rows > bt_stride) return NSA_ERR_INVALID_ARG;
            total_out += nc - f;
            prev = cu_seqlens[b];
        }
    }
    if (total_out == 0) return NSA_OK;
    const int planes = v ? 2 : 1;
    const int64_t target = (int64_t)nsm * occ;
    int chunk = (int)std::min<int64_t>(1024, std::max<int64_t>(4, (total_out * planes + target - 1) / target));

    CompressParams p;
    std::memset(&p, 0, sizeof(p));
    p.k = k;
    p.v = v;
    p.w = w;
    p.kcmp = kcmp;
    p.vcmp = vcmp;
    p.l = l;
    p.d = d;
    p.n2 = n2;
    p.d1 = d1;
    p.d2 = v ? d2 : d1;
    p.dtype = dtype == NSA_BF16 ? 0 : 1;
    p.chunk = chunk;
    p.rows_per_stage = rs;
    p.block_table = block_table;
    p.bt_stride = bt_stride;
    p.page_rows = page_rows;
    p.num_pages = (int)num_pages;
    p.tc_rows = total_out;   // rows of the contiguous outputs (all blocks when no table)
    const int threads = (int)(((rowelems / 8) + 31) / 32 * 32);

    int32_t prev_raw = 0;
    int64_t cmp_prev = 0;
    int b = 0;
    while (b < batch) {
        p.nseq = 0;
        int chunks = 0;
        for (; b < batch && p.nseq < kCompressMaxSeq; ++b) {
            const int64_t S = (int64_t)cu_seqlens[b] - prev_raw;
            const int64_t nc = ncmp_of(S, l, d);
            CompressSeq& q = p.seq[p.nseq];
            q.raw_start = prev_raw;
            q.cmp_start = (int)cmp_prev;
            q.ncmp = (int)nc;
            q.first = first_block ? first_block[b] : 0;
            q.seq = b;
            q.nchunks = (int)((nc - q.first + chunk - 1) / chunk);
            chunks += q.nchunks;
            q.chunk_end = chunks;
            prev_raw = cu_seqlens[b];
            cmp_prev += nc;
            ++p.nseq;
        }
        if (chunks == 0) continue;
        cudaError_t e = launch_compress(p, dim3(chunks, planes), threads, smem, st);
        if (e != cudaSuccess) return NSA_ERR_CUDA;
    }
    return NSA_OK;
}

extern "C" {

nsa_status_t nsa_compress(const void* k, const void* v, const void* w, int l, int d, const int32_t* cu_seqlens,
                          int batch, int n2, int d1, int d2, nsa_dtype_t dtype, void* kcmp, void* vcmp,
                          void* stream) {
    return compress_impl(k, v, w, l, d, cu_seqlens, batch, n2, d1, d2, dtype, kcmp, vcmp, stream);
}

nsa_status_t nsa_compress_paged(const void* k, const void* v, const void* w, int l, int d,
                                const int32_t* cu_seqlens, int batch, int n2, int d1, int d2, nsa_dtype_t dtype,
                                void* kcmp_pages, void* vcmp_pages, int64_t num_pages, int page_size,
                                const int32_t* block_table, int max_pages_per_seq, const int32_t* first_block,
                                void* stream) {
    if (block_table == nullptr || (reinterpret_cast<uintptr_t>(block_table) & 3u)) return NSA_ERR_INVALID_ARG;
    if (page_size < 1 || max_pages_per_seq < 1 || num_pages < 1) return NSA_ERR_INVALID_ARG;
    if (num_pages * page_size >= ((int64_t)1 << 31)) return NSA_ERR_INVALID_ARG;
    return compress_impl(k, v, w, l, d, cu_seqlens, batch, n2, d1, d2, dtype, kcmp_pages, vcmp_pages, stream,
                         first_block, block_table, max_pages_per_seq, page_size, num_pages);
}

nsa_status_t nsa_compress_status(void* stream) {
    int err = 0;
    if (read_compress_error(&err, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return NSA_ERR_CUDA;
    return error_status(err);
}

nsa_status_t nsa_compress_attention_workspace_size(int head_num, int n2, int d1, int d2, int l, int d, int lp,
                                                   int count, const int32_t* cu_seqlens_q,
                                                   const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
                                                   int batch, size_t* bytes) {
    if (bytes == nullptr) return NSA_ERR_INVALID_ARG;
    AttnPlan pl;
    nsa_status_t s = plan_attention(head_num, n2, d1, d2, l, d, lp, count, cu_seqlens_q, cu_cmp_kv, cu_sel_kv,
                                    batch, false, pl);
    if (s != NSA_OK) return s;
    *bytes = pl.ws_total;
    return NSA_OK;
}

// Steps 1-7 with the optional masks of steps 1 and 6 (null = none), already
// validated against the shapes.
static nsa_status_t compress_attention_impl(const void* q, const void* kcmp, const void* vcmp, float scale,
                                            int head_num, int l, int d, int lp, int count,
                                            const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv,
                                            const int32_t* cu_sel_kv, int batch, int n2, int d1, int d2,
                                            nsa_dtype_t dtype, const uint8_t* atten_mask, int am_s2,
                                            const uint8_t* topk_mask, int tm_s2, void* attention_out,
                                            int32_t* topk_indices, float* softmax_max, float* softmax_sum,
                                            void* workspace, size_t workspace_bytes, void* stream,
                                            int grid_cap = kMaxGrid, int npipe_max = 2, int group_begin = 0,
                                            int group_count = -1, const int32_t* block_table = nullptr,
                                            int bt_stride = 0, int page_rows = 0, int64_t num_pages = 0) {
    if (dtype != NSA_BF16 && dtype != NSA_FP16) return NSA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return NSA_ERR_INVALID_ARG;
    if (!q || !kcmp || !vcmp || !attention_out || !topk_indices || !softmax_max || !softmax_sum)
        return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kcmp) || !aligned16(vcmp) || !aligned16(attention_out) ||
        !aligned16(topk_indices) || !aligned16(softmax_max) || !aligned16(softmax_sum))
        return NSA_ERR_INVALID_ARG;
    AttnPlan pl;
    nsa_status_t s = plan_attention(head_num, n2, d1, d2, l, d, lp, count, cu_seqlens_q, cu_cmp_kv, cu_sel_kv,
                                    batch, true, pl, grid_cap, npipe_max, group_begin, group_count);
    if (s != NSA_OK) return s;
    const MaskPack mp = plan_masks(pl, cu_seqlens_q, cu_cmp_kv, cu_sel_kv, batch, atten_mask != nullptr,
                                   topk_mask != nullptr);
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        workspace_bytes < pl.ws_total + mp.am_bytes + mp.tm_bytes)
        return NSA_ERR_WORKSPACE;
    if (pl.tiles.empty()) return NSA_OK;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t t1 = cu_seqlens_q[batch - 1];
    const int64_t tc = cu_cmp_kv[batch - 1];
    CUtensorMap tq, tk, tv;
    if (block_table != nullptr) {
        // pools of pages: boxes of one page; a KV tile is NKV / page_rows pages
        if (page_rows < 8 || page_rows % 8 || pl.nkv_cols % page_rows) return NSA_ERR_UNSUPPORTED;
        if (num_pages < 1 || num_pages * page_rows >= ((int64_t)1 << 31)) return NSA_ERR_INVALID_ARG;
        if (!encode_tnd(&tq, q, dtype, d1, head_num, t1, pl.G, pl.TT) ||
            !encode_tnd(&tk, kcmp, dtype, d1, n2, num_pages * page_rows, 1, page_rows) ||
            !encode_tnd(&tv, vcmp, dtype, d2, n2, num_pages * page_rows, 1, page_rows))
            return NSA_ERR_UNSUPPORTED;
    } else if (!encode_tnd(&tq, q, dtype, d1, head_num, t1, pl.G, pl.TT) ||
               !encode_tnd(&tk, kcmp, dtype, d1, n2, tc, 1, pl.nkv_cols) ||
               !encode_tnd(&tv, vcmp, dtype, d2, n2, tc, 1, pl.nkv_cols)) {
        return NSA_ERR_UNSUPPORTED;
    }

    // workspace: [header: error word][item list][score rows][importance scratch]
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    std::vector<uint8_t> host(kWsHeader + pl.ws_tiles, 0);
    std::memcpy(host.data() + kWsHeader, pl.tiles.data(), pl.ws_tiles);
    if (cudaMemcpyAsync(ws, host.data(), host.size(), cudaMemcpyHostToDevice, st) != cudaSuccess)
        return NSA_ERR_CUDA;

    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return NSA_ERR_CUDA;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);

    AttnParams p;
    std::memset(&p, 0, sizeof(p));
    const size_t off_score = kWsHeader + ((pl.ws_tiles + 255) & ~(size_t)255);
    p.tiles = reinterpret_cast<const AttnTile*>(ws + kWsHeader);
    p.num_tiles = (int)pl.tiles.size();
    p.err = reinterpret_cast<int*>(ws);
    p.block_table = block_table;
    p.bt_stride = bt_stride;
    p.page_rows = page_rows;
    p.pool_rows = (int)(num_pages * page_rows);
    p.rows_q = t1;
    // Two passes where the head sums pay for the extra S pass: items of several
    // tokens.  With one token per item (decode) the epilogue's per-head sums are
    // short, and one pass measured faster (64 x 1 queries: 108 us against 172 us).
    p.two_pass = ((pl.G & (pl.G - 1)) == 0 && pl.G <= 32 && pl.nkv_cols == 128 && pl.max_sq > pl.TT) ? 1 : 0;
    p.score_gmem = pl.score_in_smem ? nullptr : reinterpret_cast<float*>(ws + off_score);
    p.band = reinterpret_cast<float*>(ws + off_score + pl.ws_score);
    p.capj = pl.capj;
    p.capc = pl.capc;
    p.region = pl.region;
    p.score_cap = pl.score_cap;
    p.score_in_smem = pl.score_in_smem ? 1 : 0;
    p.out = attention_out;
    p.topk = topk_indices;
    p.smax = softmax_max;
    p.ssum = softmax_sum;
    p.dtype = dtype == NSA_BF16 ? 0 : 1;
    p.n1 = head_num;
    p.n2 = n2;
    p.d1 = d1;
    p.d2 = d2;
    p.G = pl.G;
    p.tok_per_tile = pl.TT;
    p.l = l;
    p.d = d;
    p.lp = lp;
    p.count = count;
    p.a = pl.a;
    p.b = pl.b;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    p.nkv_cols = pl.nkv_cols;
    p.nslot = pl.nslot;
    p.nqbuf = pl.nqbuf;
    p.npipe = pl.npipe;
    p.nsb = pl.nsb;
    for (int i = 0; i < 2; ++i) {
        p.tm_s[i] = pl.tm_s[i];
        p.tm_o[i] = pl.tm_o[i];
    }
    p.off_q = pl.off_q;
    p.q_bytes = pl.q_bytes;
    p.off_ring = pl.off_ring;
    p.slot_bytes = pl.slot_bytes;
    p.off_rowstat = pl.off_rowstat;
    p.off_score = pl.off_score;
    p.off_bar = pl.off_bar;
    p.smem_bytes = pl.smem_bytes;
    // the masks as bit rows (one launch each, before the attention)
    uint32_t* am_bits = reinterpret_cast<uint32_t*>(ws + pl.ws_total);
    uint32_t* tm_bits = reinterpret_cast<uint32_t*>(ws + pl.ws_total + mp.am_bytes);
    if (atten_mask && launch_pack_mask(atten_mask, am_s2, (int)std::min<int64_t>(am_s2, mp.max_c), (int)mp.rows,
                                       mp.am_words, am_bits, st) != cudaSuccess)
        return NSA_ERR_CUDA;
    if (topk_mask && launch_pack_mask(topk_mask, tm_s2, (int)std::min<int64_t>(tm_s2, mp.max_s), (int)mp.rows,
                                      mp.tm_words, tm_bits, st) != cudaSuccess)
        return NSA_ERR_CUDA;
    p.am_bits = atten_mask ? am_bits : nullptr;
    p.am_words = mp.am_words;
    p.tm_bits = topk_mask ? tm_bits : nullptr;
    p.tm_words = mp.tm_words;
    const int grid = std::min(pl.grid, nsm);   // the workspace holds pl.grid CTAs' scratch
    if (launch_attention(p, tq, tk, tv, grid, st) != cudaSuccess) return NSA_ERR_CUDA;
    return NSA_OK;
}

nsa_status_t nsa_compress_attention(const void* q, const void* kcmp, const void* vcmp, float scale, int head_num,
                                    int l, int d, int lp, int count, const int32_t* cu_seqlens_q,
                                    const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv, int batch, int n2, int d1,
                                    int d2, nsa_dtype_t dtype, void* attention_out, int32_t* topk_indices,
                                    float* softmax_max, float* softmax_sum, void* workspace,
                                    size_t workspace_bytes, void* stream) {
    return compress_attention_impl(q, kcmp, vcmp, scale, head_num, l, d, lp, count, cu_seqlens_q, cu_cmp_kv,
                                   cu_sel_kv, batch, n2, d1, d2, dtype, nullptr, 0, nullptr, 0, attention_out,
                                   topk_indices, softmax_max, softmax_sum, workspace, workspace_bytes, stream);
}

nsa_status_t nsa_compress_attention_paged(const void* q, const void* kcmp_pages, const void* vcmp_pages,
                                          int64_t num_pages, int page_size, const int32_t* block_table,
                                          int max_pages_per_seq, float scale, int head_num, int l, int d, int lp,
                                          int count, const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv,
                                          const int32_t* cu_sel_kv, int batch, int n2, int d1, int d2,
                                          nsa_dtype_t dtype, void* attention_out, int32_t* topk_indices,
                                          float* softmax_max, float* softmax_sum, void* workspace,
                                          size_t workspace_bytes, void* stream) {
    if (block_table == nullptr || (reinterpret_cast<uintptr_t>(block_table) & 3u)) return NSA_ERR_INVALID_ARG;
    if (page_size < 1 || max_pages_per_seq < 1 || num_pages < 1) return NSA_ERR_INVALID_ARG;
    nsa_status_t s = check_prefix(cu_cmp_kv, batch);
    if (s != NSA_OK) return s;
    // every sequence's compressed blocks must fit its row of the block table
    for (int b = 0; b < batch; ++b) {
        const int64_t nc = cu_cmp_kv[b] - (b ? cu_cmp_kv[b - 1] : 0);
        if ((nc + page_size - 1) / page_size > max_pages_per_seq) return NSA_ERR_INVALID_ARG;
    }
    return compress_attention_impl(q, kcmp_pages, vcmp_pages, scale, head_num, l, d, lp, count, cu_seqlens_q,
                                   cu_cmp_kv, cu_sel_kv, batch, n2, d1, d2, dtype, nullptr, 0, nullptr, 0,
                                   attention_out, topk_indices, softmax_max, softmax_sum, workspace,
                                   workspace_bytes, stream, kMaxGrid, 2, 0, -1, block_table, max_pages_per_seq,
                                   page_size, num_pages);
}

nsa_status_t nsa_compress_attention_masked_workspace_size(int head_num, int n2, int d1, int d2, int l, int d,
                                                          int lp, int count, const int32_t* cu_seqlens_q,
                                                          const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
                                                          int batch, int with_atten_mask, int with_topk_mask,
                                                          size_t* bytes) {
    if (bytes == nullptr) return NSA_ERR_INVALID_ARG;
    AttnPlan pl;
    nsa_status_t s = plan_attention(head_num, n2, d1, d2, l, d, lp, count, cu_seqlens_q, cu_cmp_kv, cu_sel_kv,
                                    batch, false, pl);
    if (s != NSA_OK) return s;
    const MaskPack mp = plan_masks(pl, cu_seqlens_q, cu_cmp_kv, cu_sel_kv, batch, with_atten_mask != 0,
                                   with_topk_mask != 0);
    *bytes = pl.ws_total + mp.am_bytes + mp.tm_bytes;
    return NSA_OK;
}

nsa_status_t nsa_compress_attention_masked(const void* q, const void* kcmp, const void* vcmp, float scale,
                                           int head_num, int l, int d, int lp, int count,
                                           const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv,
                                           const int32_t* cu_sel_kv, int batch, int n2, int d1, int d2,
                                           nsa_dtype_t dtype, const uint8_t* atten_mask, int am_rows,
                                           int am_cols, const uint8_t* topk_mask, int tm_rows, int tm_cols,
                                           void* attention_out, int32_t* topk_indices, float* softmax_max,
                                           float* softmax_sum, void* workspace, size_t workspace_bytes,
                                           void* stream) {
    // every sequence's query rows and blocks must lie inside each given mask
    nsa_status_t s;
    if ((s = check_prefix(cu_seqlens_q, batch)) != NSA_OK) return s;
    if ((s = check_prefix(cu_cmp_kv, batch)) != NSA_OK) return s;
    if ((s = check_prefix(cu_sel_kv, batch)) != NSA_OK) return s;
    int64_t max_q = 0, max_c = 0, max_s = 0;
    for (int b = 0; b < batch; ++b) {
        max_q = std::max<int64_t>(max_q, cu_seqlens_q[b] - (b ? cu_seqlens_q[b - 1] : 0));
        max_c = std::max<int64_t>(max_c, cu_cmp_kv[b] - (b ? cu_cmp_kv[b - 1] : 0));
        max_s = std::max<int64_t>(max_s, cu_sel_kv[b] - (b ? cu_sel_kv[b - 1] : 0));
    }
    if (atten_mask && (am_rows < max_q || am_cols < max_c || am_cols < 1)) return NSA_ERR_INVALID_ARG;
    if (topk_mask && (tm_rows < max_q || tm_cols < max_s || tm_cols < 1)) return NSA_ERR_INVALID_ARG;
    return compress_attention_impl(q, kcmp, vcmp, scale, head_num, l, d, lp, count, cu_seqlens_q, cu_cmp_kv,
                                   cu_sel_kv, batch, n2, d1, d2, dtype, atten_mask, am_cols, topk_mask, tm_cols,
                                   attention_out, topk_indices, softmax_max, softmax_sum, workspace,
                                   workspace_bytes, stream);
}

nsa_status_t nsa_shard_groups(int n2, int world, int rank, int* group_begin, int* group_count) {
    if (n2 < 1 || world < 1 || rank < 0 || rank >= world || !group_begin || !group_count)
        return NSA_ERR_INVALID_ARG;
    // contiguous, balanced: the first n2 % world ranks take one group more
    const int q = n2 / world, r = n2 % world;
    *group_count = q + (rank < r ? 1 : 0);
    *group_begin = rank * q + std::min(rank, r);
    return NSA_OK;
}

nsa_status_t nsa_compress_attention_shard_workspace_size(int head_num, int n2, int d1, int d2, int l, int d,
                                                         int lp, int count, const int32_t* cu_seqlens_q,
                                                         const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv,
                                                         int batch, int group_begin, int group_count,
                                                         size_t* bytes) {
    if (bytes == nullptr || group_begin < 0 || group_count < 0) return NSA_ERR_INVALID_ARG;
    AttnPlan pl;
    nsa_status_t s = plan_attention(head_num, n2, d1, d2, l, d, lp, count, cu_seqlens_q, cu_cmp_kv, cu_sel_kv,
                                    batch, false, pl, kMaxGrid, 2, group_begin, group_count);
    if (s != NSA_OK) return s;
    *bytes = pl.ws_total;
    return NSA_OK;
}

nsa_status_t nsa_compress_attention_shard(const void* q, const void* kcmp, const void* vcmp, float scale,
                                          int head_num, int l, int d, int lp, int count,
                                          const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv,
                                          const int32_t* cu_sel_kv, int batch, int n2, int d1, int d2,
                                          nsa_dtype_t dtype, int group_begin, int group_count,
                                          void* attention_out, int32_t* topk_indices, float* softmax_max,
                                          float* softmax_sum, void* workspace, size_t workspace_bytes,
                                          void* stream) {
    if (group_begin < 0 || group_count < 0) return NSA_ERR_INVALID_ARG;
    return compress_attention_impl(q, kcmp, vcmp, scale, head_num, l, d, lp, count, cu_seqlens_q, cu_cmp_kv,
                                   cu_sel_kv, batch, n2, d1, d2, dtype, nullptr, 0, nullptr, 0, attention_out,
                                   topk_indices, softmax_max, softmax_sum, workspace, workspace_bytes, stream,
                                   kMaxGrid, 2, group_begin, group_count);
}

nsa_status_t nsa_compress_attention_shard_plan(int head_num, int n2, int d1, int d2, int l, int d, int lp,
                                               int count, const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv,
                                               const int32_t* cu_sel_kv, int batch, int group_begin,
                                               int group_count, int32_t* items, int64_t capacity,
                                               int64_t* n_items) {
    if (n_items == nullptr || (capacity > 0 && items == nullptr)) return NSA_ERR_INVALID_ARG;
    if (group_begin < 0 || group_count < 0) return NSA_ERR_INVALID_ARG;
    AttnPlan pl;
    nsa_status_t s = plan_attention(head_num, n2, d1, d2, l, d, lp, count, cu_seqlens_q, cu_cmp_kv, cu_sel_kv,
                                    batch, true, pl, kMaxGrid, 2, group_begin, group_count);
    if (s != NSA_OK) return s;
    *n_items = (int64_t)pl.tiles.size();
    const int64_t n = std::min<int64_t>(capacity, (int64_t)pl.tiles.size());
    for (int64_t i = 0; i < n; ++i) {
        items[3 * i + 0] = pl.tiles[i].q_row0;
        items[3 * i + 1] = pl.tiles[i].ntok;
        items[3 * i + 2] = pl.tiles[i].group;
    }
    return NSA_OK;
}

nsa_status_t nsa_select_attention_workspace_size(int head_num, int n2, int d1, int d2, int lp, int count,
                                                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv,
                                                 int batch, size_t* bytes) {
    if (bytes == nullptr) return NSA_ERR_INVALID_ARG;
    SelPlan pl;
    nsa_status_t s = plan_select(head_num, n2, d1, d2, lp, count, cu_seqlens_q, cu_seqlens_kv, batch, false, pl);
    if (s != NSA_OK) return s;
    *bytes = pl.ws_total;
    return NSA_OK;
}

nsa_status_t nsa_select_attention(const void* q, const void* k, const void* v, const int32_t* topk_indices,
                                  float scale, int head_num, int lp, int count, const int32_t* cu_seqlens_q,
                                  const int32_t* cu_seqlens_kv, int batch, int n2, int d1, int d2,
                                  nsa_dtype_t dtype, void* attention_out, float* softmax_lse, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    if (dtype != NSA_BF16 && dtype != NSA_FP16) return NSA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return NSA_ERR_INVALID_ARG;
    if (!q || !k || !v || !topk_indices || !attention_out || !softmax_lse) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(attention_out) ||
        (reinterpret_cast<uintptr_t>(topk_indices) & 3u) || (reinterpret_cast<uintptr_t>(softmax_lse) & 3u))
        return NSA_ERR_INVALID_ARG;
    SelPlan pl;
    nsa_status_t s = plan_select(head_num, n2, d1, d2, lp, count, cu_seqlens_q, cu_seqlens_kv, batch, true, pl);
    if (s != NSA_OK) return s;
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < pl.ws_total)
        return NSA_ERR_WORKSPACE;
    if (pl.tiles.empty()) return NSA_OK;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t t1 = cu_seqlens_q[batch - 1];
    const int64_t t2 = cu_seqlens_kv[batch - 1];
    CUtensorMap tq, tk, tv;
    if (!encode_tnd(&tq, q, dtype, d1, head_num, t1, pl.G, pl.TT) ||
        !encode_tnd(&tk, k, dtype, d1, n2, t2, 1, lp) || !encode_tnd(&tv, v, dtype, d2, n2, t2, 1, lp))
        return NSA_ERR_UNSUPPORTED;

    // workspace: [header: error word][tiles][list counts][list blocks][list masks]
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    std::vector<uint8_t> host(kWsHeader + pl.tiles.size() * sizeof(sel::Tile), 0);
    std::memcpy(host.data() + kWsHeader, pl.tiles.data(), pl.tiles.size() * sizeof(sel::Tile));
    if (cudaMemcpyAsync(ws, host.data(), host.size(), cudaMemcpyHostToDevice, st) != cudaSuccess)
        return NSA_ERR_CUDA;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return NSA_ERR_CUDA;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);

    sel::Params p;
    std::memset(&p, 0, sizeof(p));
    p.tiles = reinterpret_cast<const sel::Tile*>(ws + kWsHeader);
    p.num_tiles = (int)pl.tiles.size();
    p.err = reinterpret_cast<int*>(ws);
    p.rows_q = t1;
    p.topk = topk_indices;
    p.count = count;
    p.list_n = reinterpret_cast<int*>(ws + kWsHeader + pl.ws_tiles);
    p.list_blk = reinterpret_cast<int32_t*>(ws + kWsHeader + pl.ws_tiles + pl.ws_n);
    p.list_mask = reinterpret_cast<uint32_t*>(ws + kWsHeader + pl.ws_tiles + pl.ws_n + pl.ws_blk);
    p.cap = pl.cap;
    p.out = attention_out;
    p.lse = softmax_lse;
    p.dtype = dtype == NSA_BF16 ? 0 : 1;
    p.n1 = head_num;
    p.n2 = n2;
    p.d1 = d1;
    p.d2 = d2;
    p.G = pl.G;
    p.tok_per_tile = pl.TT;
    p.lp = lp;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    p.nslot = pl.nslot;
    p.nqbuf = pl.nqbuf;
    p.nsbuf = pl.nsbuf;
    p.tm_o = pl.tm_o;
    p.tm_s = pl.tm_s;
    p.s_stride = pl.s_stride;
    p.off_q = pl.off_q;
    p.q_bytes = pl.q_bytes;
    p.off_ring = pl.off_ring;
    p.slot_bytes = pl.slot_bytes;
    p.off_bar = pl.off_bar;
    p.off_x = pl.off_x;
    p.smem_bytes = pl.smem_bytes;
    if (sel::launch_plan(p, pl.max_words, st) != cudaSuccess) return NSA_ERR_CUDA;
    const int grid = std::min(pl.grid, nsm);
    if (sel::launch_attention(p, tq, tk, tv, grid, st) != cudaSuccess) return NSA_ERR_CUDA;
    return NSA_OK;
}

nsa_status_t nsa_compress_attention_backward_workspace_size(int head_num, int n2, int d1, int d2, int l, int d,
                                                            const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv,
                                                            int batch, size_t* bytes) {
    if (bytes == nullptr) return NSA_ERR_INVALID_ARG;
    BwdPlan pl;
    nsa_status_t s = plan_backward(head_num, n2, d1, d2, l, d, cu_seqlens_q, cu_cmp_kv, batch, false, pl);
    if (s != NSA_OK) return s;
    *bytes = pl.ws_total;
    return NSA_OK;
}

nsa_status_t nsa_compress_attention_backward(const void* q, const void* kcmp, const void* vcmp,
                                             const void* attention_out, const void* dout, const float* softmax_max,
                                             const float* softmax_sum, float scale, int head_num, int l, int d,
                                             const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, int batch,
                                             int n2, int d1, int d2, nsa_dtype_t dtype, float* dq, float* dkcmp,
                                             float* dvcmp, void* workspace, size_t workspace_bytes, void* stream) {
    if (dtype != NSA_BF16 && dtype != NSA_FP16) return NSA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return NSA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, kcmp, vcmp, attention_out, dout, softmax_max, softmax_sum, dq, dkcmp, dvcmp};
    for (const void* ptr : ptrs)
        if (ptr == nullptr || !aligned16(ptr)) return NSA_ERR_INVALID_ARG;
    BwdPlan pl;
    nsa_status_t s = plan_backward(head_num, n2, d1, d2, l, d, cu_seqlens_q, cu_cmp_kv, batch, true, pl);
    if (s != NSA_OK) return s;
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < pl.ws_total)
        return NSA_ERR_WORKSPACE;
    const int64_t t1 = cu_seqlens_q[batch - 1];
    const int64_t tc = cu_cmp_kv[batch - 1];
    if (t1 == 0 && tc == 0) return NSA_OK;

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    CUtensorMap tq, tdo, tk, tv;
    if (!encode_tnd(&tq, q, dtype, d1, head_num, t1, pl.G, pl.TT) ||
        !encode_tnd(&tdo, dout, dtype, d2, head_num, t1, pl.G, pl.TT) ||
        !encode_tnd(&tk, kcmp, dtype, d1, n2, tc, 1, bwd::kKV) ||
        !encode_tnd(&tv, vcmp, dtype, d2, n2, tc, 1, bwd::kKV))
        return NSA_ERR_UNSUPPORTED;

    // workspace: [header: error word][dQ items][dK/dV runs][KV tiles][row info][partial slots]
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    std::vector<uint8_t> host(pl.off_rowinfo, 0);
    auto put = [&](size_t at, const void* src, size_t n) {
        if (n) std::memcpy(host.data() + at, src, n);
    };
    put(pl.off_qitems, pl.qitems.data(), pl.qitems.size() * sizeof(bwd::QItem));
    put(pl.off_kvitems, pl.kvitems.data(), pl.kvitems.size() * sizeof(bwd::KVItem));
    put(pl.off_kvtiles, pl.kvtiles.data(), pl.kvtiles.size() * sizeof(bwd::KVTile));
    if (cudaMemcpyAsync(ws, host.data(), host.size(), cudaMemcpyHostToDevice, st) != cudaSuccess)
        return NSA_ERR_CUDA;

    bwd::Params p;
    std::memset(&p, 0, sizeof(p));
    p.qitems = reinterpret_cast<const bwd::QItem*>(ws + pl.off_qitems);
    p.n_qitems = (int)pl.qitems.size();
    p.kvitems = reinterpret_cast<const bwd::KVItem*>(ws + pl.off_kvitems);
    p.n_kvitems = (int)pl.kvitems.size();
    p.err = reinterpret_cast<int*>(ws);
    p.rowinfo = reinterpret_cast<const float2*>(ws + pl.off_rowinfo);
    p.dq = dq;
    p.part = reinterpret_cast<float*>(ws + pl.off_part);
    p.rows_q = t1;
    p.rows_c = tc;
    p.n_slots = pl.nslots;
    p.dtype = dtype == NSA_BF16 ? 0 : 1;
    p.n1 = head_num;
    p.n2 = n2;
    p.d1 = d1;
    p.d2 = d2;
    p.G = pl.G;
    p.tok_per_tile = pl.TT;
    p.l = l;
    p.d = d;
    p.scale = scale;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    p.off_row = pl.off_row;
    p.off_bar = pl.off_bar;
    p.smem_bytes = pl.smem_bytes;
    p.nst = pl.nst;
    p.stage_bytes = pl.stage_bytes;
    const int qc_bytes = ((d1 + 63) / 64) * 16384;

    if (bwd::launch_prep(attention_out, dout, softmax_max, softmax_sum,
                         reinterpret_cast<float2*>(ws + pl.off_rowinfo), t1 * head_num, d2, p.dtype,
                         st) != cudaSuccess)
        return NSA_ERR_CUDA;
    // dQ: Q and dO fixed, K/V streamed
    p.off_q = 0;
    p.off_do = qc_bytes;
    p.off_k = pl.stage_bytes;
    p.off_v = pl.stage_bytes + qc_bytes;
    if (bwd::launch_dq(p, tq, tdo, tk, tv, st) != cudaSuccess) return NSA_ERR_CUDA;
    // dK/dV: Q and dO streamed, K/V fixed
    p.off_q = 0;
    p.off_do = qc_bytes;
    p.off_k = pl.nst * pl.stage_bytes;
    p.off_v = pl.nst * pl.stage_bytes + qc_bytes;
    // dV and dK together when both accumulators fit beside the 128 score
    // columns; else one pass for each
    const int npass = pl.one_pass ? 1 : 2;
    for (int i = 0; i < npass; ++i) {
        p.mode = pl.one_pass ? 3 : 1 + i;   // bit 0 dV, bit 1 dK
        p.col_dk = pl.one_pass ? 128 : 0;
        // a second score buffer at columns 256..383 when the accumulators end by column 256
        const int acc_end = pl.one_pass ? 128 + d1 : (i == 0 ? d2 : d1);
        p.nsb = acc_end <= 256 ? 2 : 1;
        if (bwd::launch_dkdv(p, tq, tdo, tk, tv, st) != cudaSuccess) return NSA_ERR_CUDA;
    }
    if (bwd::launch_reduce(reinterpret_cast<const bwd::KVTile*>(ws + pl.off_kvtiles), (int)pl.kvtiles.size(),
                           p.part, dkcmp, dvcmp, n2, d1, d2, scale, tc, p.err, st) != cudaSuccess)
        return NSA_ERR_CUDA;
    return NSA_OK;
}

// the dw partial sums ([run][l][n2] fp32) get a fixed part of the workspace: as many runs as
// fit, up to about eight CTAs per SM
constexpr size_t kDwPartBytes = (size_t)4 << 20;

nsa_status_t nsa_compress_backward_workspace_size(const int32_t* cu_seqlens, int batch, int l, int d,
                                                  size_t* bytes) {
    if (bytes == nullptr || l < 1 || d < 1) return NSA_ERR_INVALID_ARG;
    nsa_status_t s = check_prefix(cu_seqlens, batch);
    if (s != NSA_OK) return s;
    int64_t tc = 0;
    int32_t prev = 0;
    for (int b = 0; b < batch; ++b) {
        tc += ncmp_of((int64_t)cu_seqlens[b] - prev, l, d);
        prev = cu_seqlens[b];
    }
    *bytes = kWsHeader + (((size_t)tc * 4 + 255) & ~(size_t)255) + kDwPartBytes;
    return NSA_OK;
}

nsa_status_t nsa_compress_backward(const void* k, const void* v, const void* w, const float* dkcmp,
                                   const float* dvcmp, int l, int d, const int32_t* cu_seqlens, int batch, int n2,
                                   int d1, int d2, nsa_dtype_t dtype, float* dk, float* dv, float* dw,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    // the forward's constraints (aclnnNsaCompress)
    if (dtype != NSA_BF16 && dtype != NSA_FP16) return NSA_ERR_INVALID_ARG;
    if (!k || !w || !dkcmp || !dk || !dw) return NSA_ERR_INVALID_ARG;
    const bool has_v = v != nullptr;
    if (has_v != (dvcmp != nullptr) || has_v != (dv != nullptr)) return NSA_ERR_INVALID_ARG;
    if (l % 16 || d % 16 || d < 16 || l < d || l > 128) return NSA_ERR_INVALID_ARG;
    if (n2 < 1 || d1 < 16 || d1 % 16 || d1 > 256) return NSA_ERR_INVALID_ARG;
    if (has_v && (d2 < 16 || d2 % 16 || d2 > 256)) return NSA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(dkcmp) || !aligned16(dk) ||
        (has_v && (!aligned16(v) || !aligned16(dvcmp) || !aligned16(dv))))
        return NSA_ERR_INVALID_ARG;
    size_t need = 0;
    nsa_status_t s = nsa_compress_backward_workspace_size(cu_seqlens, batch, l, d, &need);
    if (s != NSA_OK) return s;
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return NSA_ERR_WORKSPACE;
    if ((int64_t)cu_seqlens[batch - 1] * n2 * std::max(d1, has_v ? d2 : 0) > ((int64_t)1 << 40))
        return NSA_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    // first raw row of every compressed row, for the dw reduction
    std::vector<int32_t> cmp_raw;
    int32_t prev = 0;
    for (int b = 0; b < batch; ++b) {
        const int64_t nc = ncmp_of((int64_t)cu_seqlens[b] - prev, l, d);
        for (int64_t i = 0; i < nc; ++i) cmp_raw.push_back((int32_t)(prev + i * d));
        prev = cu_seqlens[b];
    }
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    std::vector<uint8_t> host(kWsHeader + cmp_raw.size() * 4, 0);
    if (!cmp_raw.empty()) std::memcpy(host.data() + kWsHeader, cmp_raw.data(), cmp_raw.size() * 4);
    if (cudaMemcpyAsync(ws, host.data(), host.size(), cudaMemcpyHostToDevice, st) != cudaSuccess)
        return NSA_ERR_CUDA;

    bwd::CompressBwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.k = k;
    p.v = v;
    p.w = w;
    p.dkcmp = dkcmp;
    p.dvcmp = dvcmp;
    p.dk = dk;
    p.dv = dv;
    p.dw = dw;
    p.cmp_raw = reinterpret_cast<const int*>(ws + kWsHeader);
    p.tc = (long long)cmp_raw.size();
    // dw runs: about eight CTAs per SM over (runs x head groups), within the partial budget
    int nruns = 0;
    if (p.tc > 0) {
        const size_t per_run = (size_t)l * n2 * 4;
        if (per_run > kDwPartBytes) return NSA_ERR_UNSUPPORTED;
        int dev = 0, nsm = 148;
        if (cudaGetDevice(&dev) != cudaSuccess) return NSA_ERR_CUDA;
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        const int hpc = bwd::compress_dw_heads_per_cta(d, n2);
        const int64_t ygroups = (n2 + hpc - 1) / hpc;
        int64_t want = std::max<int64_t>(1, (int64_t)nsm * 8 / ygroups);
        want = std::min<int64_t>(want, (int64_t)(kDwPartBytes / per_run));
        want = std::min<int64_t>(want, p.tc);
        p.dw_run = (int)((p.tc + want - 1) / want);
        nruns = (int)((p.tc + p.dw_run - 1) / p.dw_run);
    }
    p.dw_part = reinterpret_cast<float*>(ws + kWsHeader + ((cmp_raw.size() * 4 + 255) & ~(size_t)255));
    p.t2 = cu_seqlens[batch - 1];
    p.l = l;
    p.d = d;
    p.n2 = n2;
    p.d1 = d1;
    p.d2 = has_v ? d2 : 0;
    p.dtype = dtype == NSA_BF16 ? 0 : 1;

    // dk, dv: sequences in batches of the parameter block's capacity
    prev = 0;
    int64_t cmp_prev = 0;
    int b = 0;
    while (b < batch) {
        p.nseq = 0;
        int blocks = 0;
        for (; b < batch && p.nseq < kCompressMaxSeq; ++b) {
            const int64_t S = (int64_t)cu_seqlens[b] - prev;
            const int64_t nc = ncmp_of(S, l, d);
            bwd::CompressBwdSeq& q = p.seq[p.nseq];
            q.raw_start = prev;
            q.raw_len = (int)S;
            q.cmp_start = (int)cmp_prev;
            q.n_cmp = (int)nc;
            blocks += (int)((S + bwd::kRowsPerCta - 1) / bwd::kRowsPerCta);
            q.blk_end = blocks;
            prev = cu_seqlens[b];
            cmp_prev += nc;
            ++p.nseq;
        }
        if (blocks > 0 && bwd::launch_compress_bwd_dx(p, blocks, st) != cudaSuccess) return NSA_ERR_CUDA;
    }
    if (bwd::launch_compress_bwd_dw(p, nruns, st) != cudaSuccess) return NSA_ERR_CUDA;
    return NSA_OK;
}

nsa_status_t nsa_workspace_status(const void* workspace, void* stream) {
    if (workspace == nullptr) return NSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return NSA_ERR_CUDA;
    int err = 0;
    if (cudaMemcpy(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return NSA_ERR_CUDA;
    return error_status(err);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Variant with a fixed, library-owned scratch area (no counterpart on the
// source pages).  Some callers cannot allocate device memory at all: a host
// application that has already reserved nearly all of the GPU's memory for
// its own pools, a plugin whose host environment hands it only the tensors
// it works on, or a latency-critical path where an allocation call is not
// allowed.  They pass only inputs and outputs; the workspace lives in this
// file-scope array, which every GPU that loads the library holds until the
// process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB per device
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[256] = {};   // device address of g_static_scratch, per device ordinal

}  // namespace

extern "C" nsa_status_t nsa_compress_attention_noalloc(
    const void* q, const void* kcmp, const void* vcmp, float scale, int head_num, int l, int d, int lp,
    int count, const int32_t* cu_seqlens_q, const int32_t* cu_cmp_kv, const int32_t* cu_sel_kv, int batch,
    int n2, int d1, int d2, nsa_dtype_t dtype, void* attention_out, int32_t* topk_indices,
    float* softmax_max, float* softmax_sum, void* stream) {
    AttnPlan pl;
    nsa_status_t s = plan_attention(head_num, n2, d1, d2, l, d, lp, count, cu_seqlens_q, cu_cmp_kv, cu_sel_kv,
                                    batch, false, pl);
    if (s != NSA_OK) return s;
    int grid_cap = kMaxGrid, npipe_max = 2;
    if (pl.ws_total > kStaticScratchBytes) {
        // the per-CTA scratch of the full grid does not fit the fixed array: run
        // fewer persistent CTAs, then one M-tile per item, before refusing
        bool fit = false;
        for (int np = pl.npipe; np >= 1 && !fit; --np) {
            AttnPlan q;
            if (plan_attention(head_num, n2, d1, d2, l, d, lp, count, cu_seqlens_q, cu_cmp_kv, cu_sel_kv, batch,
                               false, q, kMaxGrid, np) != NSA_OK ||
                q.ws_fixed >= kStaticScratchBytes || q.ws_per_cta == 0)
                continue;
            const size_t n = (kStaticScratchBytes - q.ws_fixed) / q.ws_per_cta;
            if (n >= 1) {
                grid_cap = (int)std::min<size_t>(n, kMaxGrid);
                npipe_max = np;
                fit = true;
            }
        }
        if (!fit) return NSA_ERR_WORKSPACE;   // one CTA's scratch exceeds the fixed array
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return NSA_ERR_CUDA;
    void* scratch = nullptr;
    {
        // first call on a device: look up the device address of the array with
        // that device current (host code may not use the symbol itself)
        std::lock_guard<std::mutex> lk(g_scratch_mu);
        if (g_scratch_addr[dev] == nullptr) {
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr)
                return NSA_ERR_CUDA;
            g_scratch_addr[dev] = ptr;
        }
        scratch = g_scratch_addr[dev];
    }
    // the regular entry point rewrites the scratch header (error word = 0) and
    // the tile list on every call before its kernel runs
    return compress_attention_impl(q, kcmp, vcmp, scale, head_num, l, d, lp, count, cu_seqlens_q, cu_cmp_kv,
                                   cu_sel_kv, batch, n2, d1, d2, dtype, nullptr, 0, nullptr, 0, attention_out,
                                   topk_indices, softmax_max, softmax_sum, scratch, kStaticScratchBytes, stream,
                                   grid_cap, npipe_max);
}

// Error word of the last nsa_compress_attention_noalloc on the current device:
// the first int of the fixed scratch array, read after `stream` has drained.
extern "C" nsa_status_t nsa_noalloc_status(void* stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return NSA_ERR_CUDA;
    int err = 0;
    if (cudaMemcpyFromSymbol(&err, g_static_scratch, sizeof(int), 0, cudaMemcpyDeviceToHost) != cudaSuccess)
        return NSA_ERR_CUDA;
    return error_status(err);
}
