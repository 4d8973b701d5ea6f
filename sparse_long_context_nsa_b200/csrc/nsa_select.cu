// nsa_select.cu -- selection attention (sm_100a): block-sparse attention over
// the l'-token blocks of raw K/V that the compressed branch's top-k lists per
// query row and KV group.
//
// "lite_boost.ops.rain_fusion_attention": attention restricted to the KV
// blocks listed per query block and head (select_idx: ascending valid
// indices, then -1 padding), causal mask (mask_type 0), GQA through
// num_key_value_heads, outputs attention_out and softmax_lse.  Here a query
// block is one token and the list is the top-k row of (token, KV group) from
// nsa_compress_attention.  Query row t_loc of a sequence sits at key
// position t = t_loc + (S_kv - S_q); it attends to the keys p of its listed
// blocks (block j holds p = j l' .. j l' + l' - 1) with p <= t and p < S_kv.
//
// Two kernels:
//   sel_plan_kernel  one CTA per M-tile (128/G tokens x the G heads of one KV
//                    group): the union of the tiles' listed blocks, ascending,
//                    and per block a bit mask of the tokens that listed it.
//   sel_attn_kernel  tcgen05 attention over those blocks, one KV tile of l'
//                    keys per listed block, with a one-pass online softmax:
//                    S = Q K^T into tensor memory, P = 2^(s*scale*log2e - m)
//                    written back over S, O += P V; a row masks the columns
//                    of a block it did not list and the causal / sequence-end
//                    columns; O / L and softmax_lse at the end of the tile.
// Warp roles (192 threads): warps 0-3 softmax and output (one tile row per
// thread), warp 4 TMA producer, warp 5 MMA issuer and tensor-memory owner.
// Every mbarrier wait is bounded; a timeout sets the workspace error word and
// every role drains.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "nsa_internal.h"
#include "ptx.cuh"

namespace nsa {
namespace sel {

enum BarId {
    B_Q_FULL0 = 0,                        // + Q buffer (2)
    B_Q_EMPTY0 = B_Q_FULL0 + 2,           // + Q buffer (2)
    B_S_FULL0 = B_Q_EMPTY0 + 2,           // + score buffer: S = Q K^T landed
    B_S_EMPTY0 = B_S_FULL0 + kMaxSBuf,    // + score buffer: the P V reading it retired
    B_P_FULL0 = B_S_EMPTY0 + kMaxSBuf,    // + score buffer: P written (4 warps)
    B_O_FULL = B_P_FULL0 + kMaxSBuf,
    B_O_EMPTY,
    B_MMA_DONE,
    B_SLOT_FULL0,                         // + slot (8)
    B_SLOT_EMPTY0 = B_SLOT_FULL0 + 8,
    B_COUNT = B_SLOT_EMPTY0 + 8
};
static_assert(8 * B_COUNT + 8 <= kBarBytes, "barrier area");

template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// Block lists.  The listed blocks of the tile's tokens are marked in a bit map
// over the sequence's blocks (-1 and blocks past the sequence are skipped, a
// repeat marks the same bit); the set bits, in order, are the tile's list, and
// a second sweep over the (token, block) pairs sets each token's bit in the
// mask of its blocks.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPlanThreads)
sel_plan_kernel(const Params p) {
    extern __shared__ uint32_t plan_smem[];
    const Tile t = p.tiles[blockIdx.x];
    const int nw = (t.n_blk + 31) / 32;
    uint32_t* bitmap = plan_smem;            // nw words
    uint32_t* woff = plan_smem + nw;         // exclusive prefix of the set bits per word
    __shared__ int part[kPlanThreads];
    const int tid = threadIdx.x;
    for (int w = tid; w < nw; w += kPlanThreads) bitmap[w] = 0u;
    __syncthreads();
    const int npair = t.ntok * p.count;
    auto listed = [&](int idx, int& tau) {
        tau = idx / p.count;
        const int c = idx - tau * p.count;
        const int j = p.topk[((size_t)(t.q_row0 + tau) * p.n2 + t.group) * p.count + c];
        return (j >= 0 && j < t.n_blk) ? j : -1;
    };
    for (int idx = tid; idx < npair; idx += kPlanThreads) {
        int tau;
        const int j = listed(idx, tau);
        if (j >= 0) atomicOr(&bitmap[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    // prefix of the set bits: thread tid owns words [w0, w1)
    const int per = (nw + kPlanThreads - 1) / kPlanThreads;
    const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bitmap[w]);
    part[tid] = cnt;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int i = 0; i < kPlanThreads; ++i) {
            const int c = part[i];
            part[i] = run;
            run += c;
        }
        p.list_n[blockIdx.x] = run;
    }
    __syncthreads();
    int32_t* blk = p.list_blk + (size_t)blockIdx.x * p.cap;
    uint32_t* msk = p.list_mask + (size_t)blockIdx.x * p.cap * 4;
    int pos = part[tid];
    for (int w = w0; w < w1; ++w) {
        woff[w] = (uint32_t)pos;
        uint32_t bits = bitmap[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            blk[pos] = w * 32 + b;
            msk[4 * pos + 0] = msk[4 * pos + 1] = msk[4 * pos + 2] = msk[4 * pos + 3] = 0u;
            ++pos;
            bits &= bits - 1u;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < npair; idx += kPlanThreads) {
        int tau;
        const int j = listed(idx, tau);
        if (j < 0) continue;
        const int q = (int)woff[j >> 5] + __popc(bitmap[j >> 5] & ((1u << (j & 31)) - 1u));
        atomicOr(&msk[4 * q + (tau >> 5)], 1u << (tau & 31));
    }
}

cudaError_t launch_plan(const Params& p, int max_words, cudaStream_t st) {
    const size_t smem = (size_t)max_words * 8;
    cudaError_t e = cudaFuncSetAttribute(sel_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    sel_plan_kernel<<<p.num_tiles, kPlanThreads, smem, st>>>(p);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Attention over the listed blocks.  LP = l' keys per KV tile.
//
// A KV tile holds BPT listed blocks side by side (NKV = BPT * l' keys).  One
// pass with an online softmax per row: the row's reference maximum m moves
// up only when a KV tile's maximum exceeds it by more than 8 (exponent units,
// base 2): P = 2^(x - m) then stays at most 2^8, and O and L are rescaled by
// 2^(m_old - m_new) only at those moves.  O / L and the log-sum-exp are
// formed once per M-tile.  P is written, in the storage dtype, over the first
// NKV/2 columns of the score buffer it came from; the buffer is reused once
// the P V that reads it has retired.  A warp none of whose rows attend to a
// KV tile skips the exponentials and writes zero P.
// ---------------------------------------------------------------------------
template <typename T, int LP>
__global__ void __launch_bounds__(attn_threads(LP), 1)
sel_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const Params p) {
    // BPT listed blocks side by side in one KV tile of NKV keys
    constexpr int BPT = blocks_per_tile(LP);
    // a KV tile of several listed blocks splits between two softmax warps per lane quadrant
    constexpr bool kSplit = attn_split(LP);
    constexpr int kSoft = kSplit ? 8 : 4;   // softmax warps
    constexpr int NKV = BPT * LP;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr int kWarpTma = 4, kWarpMma = 5;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + p.off_bar + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.off_bar + 8 * B_COUNT + 4);
    auto bar = [&](int id) { return smem_u32(&bars[id]); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.G;
    const int TT = p.tok_per_tile;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(B_Q_FULL0 + i), 1);
            mbar_init(bar(B_Q_EMPTY0 + i), 1);
        }
        for (int i = 0; i < kMaxSBuf; ++i) {
            mbar_init(bar(B_S_FULL0 + i), 1);
            mbar_init(bar(B_S_EMPTY0 + i), 1);
            mbar_init(bar(B_P_FULL0 + i), kSoft);
        }
        mbar_init(bar(B_O_FULL), 1);
        mbar_init(bar(B_O_EMPTY), kSoft);
        mbar_init(bar(B_MMA_DONE), 1);
        for (int s = 0; s < 8; ++s) {
            mbar_init(bar(B_SLOT_FULL0 + s), 1);
            mbar_init(bar(B_SLOT_EMPTY0 + s), 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + p.tm_o;

    const uint32_t q_addr0 = smem_u32(smem + p.off_q);
    const uint32_t ring_addr = smem_u32(smem + p.off_ring);
    const int nslot = p.nslot;
    const int nqbuf = p.nqbuf;
    const int nsbuf = p.nsbuf;
    const int nqc = (p.d1 + 63) / 64;    // 64-element chunks of a Q/K row
    const int nvc = (p.d2 + 63) / 64;    // 64-element chunks of a V row
    // tensor-memory column of score buffer sb
    auto s_col = [&](uint32_t sb) { return (uint32_t)p.tm_s + sb * (uint32_t)p.s_stride; };
    // the block list of tile `tile` (written by sel_plan_kernel)
    auto list_n = [&](int tile) { return min(p.list_n[tile], p.cap); };
    auto list_blk = [&](int tile, int i) { return p.list_blk[(size_t)tile * p.cap + i]; };
    // KV tile i of a tile holds its listed blocks i*BPT .. i*BPT+BPT-1 (a
    // slot past the list repeats the tile's first block and is masked).
    // Every role walks the same tiles and counts them alike: a tile with an
    // empty list takes no Q, no K/V and no MMA, and is not counted in qc / oc.
    // A tile's KV tiles are consumed in the order S_0 .. S_{min(nkv,nsbuf)-1},
    // then for i = 0 .. nkv-1: P V_i, and S_{i-lag+nsbuf} once i >= lag.  S_j
    // thus lands nsbuf - lag steps before its P V is due, and a buffer is
    // refilled lag steps after the P V that frees it was issued.
    const int lag = max(1, nsbuf / 2);

    if (warp == kWarpTma) {
        // ============================ TMA producer ============================
        if (lane == 0) {
            uint32_t item = 0, qc = 0;
            const uint32_t q_bytes = (uint32_t)(nqc * 64 * G * TT * 2);
            const uint32_t k_bytes = (uint32_t)(nqc * 64 * NKV * 2);
            const uint32_t v_bytes = (uint32_t)(nvc * 64 * NKV * 2);
            bool ok = true;
            // K or V of KV tile i: block q of the tile to rows q*LP.. of each
            // 64-column chunk
            auto load_kv = [&](bool is_v, int tile, const Tile& t, int n, int i) {
                const int slot = item % nslot;
                const uint32_t ph = (item / nslot) & 1;
                ok = ok && mbar_wait(bar(B_SLOT_EMPTY0 + slot), ph ^ 1, abort_flag, p.err, kErrTimeoutBase + 2);
                if (!ok) return;
                const uint32_t fb = bar(B_SLOT_FULL0 + slot);
                const uint32_t dst = ring_addr + slot * p.slot_bytes;
                mbar_arrive_expect_tx(fb, is_v ? v_bytes : k_bytes);
                const int nc = is_v ? nvc : nqc;
                for (int q = 0; q < BPT; ++q) {
                    const int e = (i * BPT + q < n) ? i * BPT + q : i * BPT;
                    const int row = t.kv_row0 + list_blk(tile, e) * LP;
                    for (int c = 0; c < nc; ++c)
                        tma_load_3d(dst + c * NKV * 128 + q * LP * 128, is_v ? &tm_v : &tm_k, c * 64, t.group, row,
                                    fb);
                }
                ++item;
            };
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                const int n = list_n(tile);
                if (n == 0) continue;
                const Tile t = p.tiles[tile];
                const int qb = qc % nqbuf;
                ok = mbar_wait(bar(B_Q_EMPTY0 + qb), ((qc / nqbuf) & 1) ^ 1, abort_flag, p.err,
                               kErrTimeoutBase + 3);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(B_Q_FULL0 + qb), q_bytes);
                const uint32_t qdst = q_addr0 + qb * p.q_bytes;
                for (int c = 0; c < nqc; ++c)
                    tma_load_3d(qdst + c * 16384, &tm_q, c * 64, t.group * G, t.q_row0, bar(B_Q_FULL0 + qb));
                const int nkv = (n + BPT - 1) / BPT;
                const int npro = min(nkv, nsbuf);
                for (int i = 0; i < npro && ok; ++i) load_kv(false, tile, t, n, i);
                for (int i = 0; i < nkv && ok; ++i) {
                    load_kv(true, tile, t, n, i);
                    if (i >= lag && i - lag + nsbuf < nkv) load_kv(false, tile, t, n, i - lag + nsbuf);
                }
                ++qc;
            }
        }
    } else if (warp == kWarpMma) {
        // ============================ MMA issuer =============================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_f16(kBF16, 128, NKV, false, false);
            const uint32_t idesc_pv = idesc_f16(kBF16, 128, p.d2, false, true);
            const int nks_qk = p.d1 / 16;
            constexpr int nks_pv = NKV / 16;
            uint32_t item = 0, scnt = 0, qc = 0, oc = 0;
            bool ok = true;
            uint32_t q_addr = q_addr0;
            // S = Q K^T of the next block into its score buffer, once the P V
            // that last read the buffer has retired
            auto issue_s = [&]() {
                const uint32_t sb = scnt % nsbuf;
                ok = ok && mbar_wait(bar(B_S_EMPTY0 + sb), ((scnt / nsbuf) & 1) ^ 1, abort_flag, p.err,
                                     kErrTimeoutBase + 4);
                const int slot = item % nslot;
                ok = ok && mbar_wait(bar(B_SLOT_FULL0 + slot), (item / nslot) & 1, abort_flag, p.err,
                                     kErrTimeoutBase + 5);
                if (!ok) return;
                tc_fence_after();
                const uint32_t kbase = ring_addr + slot * p.slot_bytes;
                for (int ks = 0; ks < nks_qk; ++ks) {
                    const uint32_t off = (ks & 3) * 32;   // 16 elements inside a 128-byte row
                    const uint64_t bd = sdesc_sw128(kbase + (ks >> 2) * (NKV * 128) + off, 16, 1024);
                    const uint64_t ad = sdesc_sw128(q_addr + (ks >> 2) * 16384 + off, 16, 1024);
                    umma_ss(tmem + s_col(sb), ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
                }
                umma_commit(bar(B_S_FULL0 + sb));
                umma_commit(bar(B_SLOT_EMPTY0 + slot));
                ++item;
                ++scnt;
            };
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
                const int n = list_n(tile);
                if (n == 0) continue;
                const int qb = qc % nqbuf;
                ok = mbar_wait(bar(B_Q_FULL0 + qb), (qc / nqbuf) & 1, abort_flag, p.err, kErrTimeoutBase + 6);
                if (!ok) break;
                tc_fence_after();
                q_addr = q_addr0 + qb * p.q_bytes;
                const uint32_t s0 = scnt;               // running index of the tile's KV tile 0
                const int nkv = (n + BPT - 1) / BPT;
                const int npro = min(nkv, nsbuf);
                for (int i = 0; i < npro && ok; ++i) issue_s();
                for (int i = 0; i < nkv && ok; ++i) {
                    const uint32_t gi = s0 + i;
                    const uint32_t sb = gi % nsbuf;
                    // O of the previous tile has been read out before P V_0 overwrites it
                    if (i == 0)
                        ok = ok && mbar_wait(bar(B_O_EMPTY), (oc & 1) ^ 1, abort_flag, p.err,
                                             kErrTimeoutBase + 7);
                    ok = ok && mbar_wait(bar(B_P_FULL0 + sb), (gi / nsbuf) & 1, abort_flag, p.err,
                                         kErrTimeoutBase + 8);
                    const int slot = item % nslot;
                    ok = ok && mbar_wait(bar(B_SLOT_FULL0 + slot), (item / nslot) & 1, abort_flag, p.err,
                                         kErrTimeoutBase + 9);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t vbase = ring_addr + slot * p.slot_bytes;
#pragma unroll
                    for (int ks = 0; ks < nks_pv; ++ks) {
                        const uint64_t bd = sdesc_sw128(vbase + ks * 2048, NKV * 128, 1024);
                        // split tiles: the second half's P sits at the start of its own half
                        const uint32_t pc = ks * 8 + ((kSplit && ks >= nks_pv / 2) ? NKV / 4 : 0);
                        umma_ts(tmem_o, tmem + s_col(sb) + pc, bd, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(bar(B_S_EMPTY0 + sb));     // the buffer is free, O holds P V_0..i
                    umma_commit(bar(B_SLOT_EMPTY0 + slot));
                    ++item;
                    // refill the buffer of block i - lag: its P V was issued lag
                    // steps ago and has had that long to retire
                    if (i >= lag && i - lag + nsbuf < nkv) issue_s();
                }
                if (!ok) break;
                umma_commit(bar(B_O_FULL));
                umma_commit(bar(B_Q_EMPTY0 + qb));
                ++qc;
                ++oc;
            }
            // every MMA issued so far has retired before the tensor memory is freed
            umma_commit(bar(B_MMA_DONE));
            mbar_wait(bar(B_MMA_DONE), 0, abort_flag, nullptr, 0);
        }
    } else if (warp < 4 || (kSplit && warp >= 6 && warp < 10)) {
        // ===== softmax and output (one row per thread; split tiles: two warps per row) =====
        // warps 0-3 take the first NKV/2 columns of a KV tile (all of it when the tile does
        // not split), warps 6-9 the second, in lane quadrant warp % 4.  The two halves of a
        // row exchange their maxima through shared memory every tile (both then move the
        // reference maximum alike) and their sums once per M-tile.
        constexpr int NH = kSplit ? NKV / 2 : NKV;   // columns per warp
        const int quad = warp & 3, half = warp >= 6 ? 1 : 0;
        const int col0 = half * NH;
        const int row = quad * 32 + lane;          // tile row = TMEM lane
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float* const xmax = reinterpret_cast<float*>(smem + p.off_x);        // [parity][half][128]
        float* const xsum = xmax + 2 * 2 * 128;                               // [half][128]
        const float c2 = p.scale_log2;
        const int h = row % G;
        const int tok = row / G;
        // scores in "exponent units": x = s * ce.  With a positive scale the
        // raw scores are used as they are (ce = c2); a zero or negative scale
        // first multiplies them in (ce = 1).  Key k of block q of the KV tile
        // is attended to iff k < lim[q]; the others become -inf.
        const bool pos_scale = c2 > 0.f;
        const float ce = pos_scale ? c2 : 1.f;
        auto prep = [&](float (&s)[NH], const int (&lim)[BPT]) {
            if (!pos_scale) {
#pragma unroll
                for (int c = 0; c < NH; ++c) s[c] *= c2;
            }
            bool full = true;
#pragma unroll
            for (int q = 0; q < BPT; ++q) full = full && lim[q] == LP;
            if (!full) {
#pragma unroll
                for (int c = 0; c < NH; ++c) {
                    const int cg = col0 + c;   // column of the KV tile
                    s[c] = (cg % LP < lim[cg / LP]) ? s[c] : -INFINITY;
                }
            }
        };
        // the two warps of a lane quadrant meet at named barrier 1 + quad
        auto pair_sync = [&]() {
            if constexpr (kSplit) named_bar_sync(1 + quad, 64);
        };
        // this warp's O columns: its half of the 16-column pieces
        const int npc = p.d2 / 16;
        const int oc0 = kSplit ? half * ((npc + 1) / 2) * 16 : 0;
        const int oc1 = kSplit ? min(p.d2, (half + 1) * ((npc + 1) / 2) * 16) : p.d2;
        uint32_t scnt = 0, oc = 0;

        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
            const Tile t = p.tiles[tile];
            const int n = list_n(tile);
            const bool valid = (row < TT * G) && (tok < t.ntok) &&
                               nsa_index_ok(t.q_row0 + tok < p.rows_q, p.err, 7);
            const size_t ridx = (size_t)(t.q_row0 + tok) * p.n1 + (size_t)t.group * G + h;
            T* orow = reinterpret_cast<T*>(p.out) + ridx * p.d2;
            if (n == 0) {
                // no listed block: nothing is attended to
                if (valid) {
                    if (half == 0) p.lse[ridx] = -INFINITY;
                    for (int c = oc0; c < oc1; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0u, 0u, 0u, 0u);
                }
                continue;
            }
            const int tpos = t.t0 + tok;
            // list entry e: its block and the mask word of this row's token (a
            // zero word past the list).  The entries of KV tile i + 2 are read
            // while tile i is processed, so that their latency is hidden.
            auto fetch = [&](int e, int& b, uint32_t& w) {
                b = (e < n) ? list_blk(tile, e) : 0;
                w = (e < n) ? p.list_mask[((size_t)tile * p.cap + e) * 4 + (tok >> 5)] : 0u;
            };
            // keys of the block this row attends to: a prefix, cut by the causal
            // rule and the end of the sequence; none when its token did not
            // list the block
            auto lim_of = [&](int b, uint32_t w) {
                if (!valid || !((w >> (tok & 31)) & 1u)) return 0;
                const int lim = min(LP, min(tpos - b * LP + 1, t.s_kv - b * LP));
                return lim > 0 ? lim : 0;
            };

            float m = -INFINITY, L = 0.f;   // reference max (exponent units), this half's sum of 2^(x - m)
            const int nkv = (n + BPT - 1) / BPT;
            int lim[BPT], nb[BPT];
            uint32_t nw[BPT];
#pragma unroll
            for (int q = 0; q < BPT; ++q) {
                int b0;
                uint32_t w0;
                fetch(q, b0, w0);
                lim[q] = lim_of(b0, w0);
                fetch(BPT + q, nb[q], nw[q]);
            }
            for (int i = 0; i < nkv; ++i) {
                const uint32_t sb = scnt % nsbuf;
                const uint32_t ts = tmem + lane_off + s_col(sb) + col0;
                int lim_next[BPT];
                bool any = false;
#pragma unroll
                for (int q = 0; q < BPT; ++q) {
                    lim_next[q] = lim_of(nb[q], nw[q]);
                    fetch((i + 2) * BPT + q, nb[q], nw[q]);
                    const bool mine = !kSplit || (q * LP < col0 + NH && (q + 1) * LP > col0);
                    any = any || (mine && lim[q] > 0);
                }
                const bool work = __any_sync(0xffffffffu, any);
                mbar_wait(bar(B_S_FULL0 + sb), (scnt / nsbuf) & 1, abort_flag, p.err, kErrTimeoutBase + 10);
                tc_fence_after();
                uint32_t pw[NH / 2];
                float s[NH];
                float mx = -INFINITY;
                if (work) {
                    {
                        uint32_t r[NH];
                        tmem_ld_cols<NH>(ts, r);
                        tmem_wait_ld_regs<NH>(r);
#pragma unroll
                        for (int c = 0; c < NH; ++c) s[c] = __uint_as_float(r[c]);
                    }
                    prep(s, lim);
                    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < NH; c += 8) {
                        mx4[0] = fmax3(mx4[0], s[c + 0], s[c + 1]);
                        mx4[1] = fmax3(mx4[1], s[c + 2], s[c + 3]);
                        mx4[2] = fmax3(mx4[2], s[c + 4], s[c + 5]);
                        mx4[3] = fmax3(mx4[3], s[c + 6], s[c + 7]);
                    }
                    mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * ce;
                }
                if constexpr (kSplit) {
                    // the row's maximum over both halves (buffers alternate by tile, so a
                    // write never meets the other warp's read of the tile before)
                    float* xm = xmax + (scnt & 1) * 256;
                    xm[half * 128 + row] = mx;
                    pair_sync();
                    mx = fmaxf(mx, xm[(half ^ 1) * 128 + row]);
                }
                // move the reference up only by more than 8: P <= 2^8 in between
                const bool raise = mx > m + 8.f;            // from -inf: any finite maximum
                const bool resc = raise && (m != -INFINITY); // O holds earlier blocks' P V
                float corr = 1.f;
                if (raise) {
                    corr = ex2(m - mx);                     // 0 from -inf
                    L *= corr;
                    m = mx;
                }
                if (__any_sync(0xffffffffu, resc)) {
                    // this warp's O columns times corr, after P V of the previous block
                    const uint32_t pg = scnt - 1;
                    mbar_wait(bar(B_S_EMPTY0 + pg % nsbuf), (pg / nsbuf) & 1, abort_flag, p.err,
                              kErrTimeoutBase + 11);
                    tc_fence_after();
                    const float f = resc ? corr : 1.f;
                    for (int c = oc0; c < oc1; c += 16) {
                        uint32_t r[16];
                        tmem_ld16(tmem_o + lane_off + c, r);
                        tmem_wait_ld_regs<16>(r);
#pragma unroll
                        for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
                        tmem_st16(tmem_o + lane_off + c, r);
                    }
                }
                if (work) {
                    const float mref = (m == -INFINITY) ? 0.f : m;
                    const float2 ce2 = make_float2(ce, ce), nm2 = make_float2(-mref, -mref);
                    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                     make_float2(0.f, 0.f)};
#pragma unroll
                    for (int c = 0; c < NH; c += 2) {
                        const float2 x = ffma2(make_float2(s[c], s[c + 1]), ce2, nm2);
                        const float2 e2 = make_float2(ex2(x.x), ex2(x.y));
                        acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], e2);
                        pw[c >> 1] = pack2<T>(e2.x, e2.y);
                    }
                    const float2 t01 = fadd2(acc[0], acc[1]), t23 = fadd2(acc[2], acc[3]);
                    L += (t01.x + t01.y) + (t23.x + t23.y);
                } else {
#pragma unroll
                    for (int c = 0; c < NH / 2; ++c) pw[c] = 0u;
                }
                // P in the storage dtype over the first NH/2 columns of this warp's part of
                // the buffer (columns it has read)
                if constexpr ((NH / 2) % 16 == 0) {
#pragma unroll
                    for (int c = 0; c < NH / 32; ++c) tmem_st16(ts + c * 16, pw + c * 16);
                } else {
#pragma unroll
                    for (int c = 0; c < NH / 16; ++c) tmem_st8(ts + c * 8, pw + c * 8);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_P_FULL0 + sb));
                ++scnt;
#pragma unroll
                for (int q = 0; q < BPT; ++q) lim[q] = lim_next[q];
            }
            if constexpr (kSplit) {
                // the row's sum over both halves
                xsum[half * 128 + row] = L;
                pair_sync();
                L += xsum[(half ^ 1) * 128 + row];
                pair_sync();   // both have read before the next M-tile writes again
            }

            // ------------- O / L -> attention_out, log-sum-exp -------------
            mbar_wait(bar(B_O_FULL), oc & 1, abort_flag, p.err, kErrTimeoutBase + 12);
            tc_fence_after();
            if (valid && half == 0) p.lse[ridx] = (L > 0.f) ? (m + lg2(L)) * 0.69314718055994530942f : -INFINITY;
            const float inv = (L > 0.f) ? 1.f / L : 0.f;
            for (int c = oc0; c < oc1; c += 16) {
                uint32_t r[16];
                tmem_ld16(tmem_o + lane_off + c, r);
                tmem_wait_ld_regs<16>(r);
                if (valid) {
                    uint4 w0, w1;
                    w0.x = pack2<T>(__uint_as_float(r[0]) * inv, __uint_as_float(r[1]) * inv);
                    w0.y = pack2<T>(__uint_as_float(r[2]) * inv, __uint_as_float(r[3]) * inv);
                    w0.z = pack2<T>(__uint_as_float(r[4]) * inv, __uint_as_float(r[5]) * inv);
                    w0.w = pack2<T>(__uint_as_float(r[6]) * inv, __uint_as_float(r[7]) * inv);
                    w1.x = pack2<T>(__uint_as_float(r[8]) * inv, __uint_as_float(r[9]) * inv);
                    w1.y = pack2<T>(__uint_as_float(r[10]) * inv, __uint_as_float(r[11]) * inv);
                    w1.z = pack2<T>(__uint_as_float(r[12]) * inv, __uint_as_float(r[13]) * inv);
                    w1.w = pack2<T>(__uint_as_float(r[14]) * inv, __uint_as_float(r[15]) * inv);
                    *reinterpret_cast<uint4*>(orow + c) = w0;
                    *reinterpret_cast<uint4*>(orow + c + 8) = w1;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_O_EMPTY));
            ++oc;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) {
        // a wait gave up: give copies and MMAs still in flight time to land
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 20000000ull) {
        }
    }
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <typename T, int LP>
static cudaError_t launch_t(const Params& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            int grid, cudaStream_t st) {
    auto kern = sel_attn_kernel<T, LP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, attn_threads(LP), p.smem_bytes, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_lp(const Params& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             int grid, cudaStream_t st) {
    switch (p.lp) {
        case 16: return launch_t<T, 16>(p, tq, tk, tv, grid, st);
        case 32: return launch_t<T, 32>(p, tq, tk, tv, grid, st);
        case 48: return launch_t<T, 48>(p, tq, tk, tv, grid, st);
        case 64: return launch_t<T, 64>(p, tq, tk, tv, grid, st);
        case 80: return launch_t<T, 80>(p, tq, tk, tv, grid, st);
        case 96: return launch_t<T, 96>(p, tq, tk, tv, grid, st);
        case 112: return launch_t<T, 112>(p, tq, tk, tv, grid, st);
        case 128: return launch_t<T, 128>(p, tq, tk, tv, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_attention(const Params& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             int grid, cudaStream_t st) {
    return p.dtype == 0 ? launch_lp<__nv_bfloat16>(p, tq, tk, tv, grid, st)
                        : launch_lp<__half>(p, tq, tk, tv, grid, st);
}

}  // namespace sel
}  // namespace nsa
