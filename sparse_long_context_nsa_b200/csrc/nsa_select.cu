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
//   sel_attn_kernel  the two-pass tcgen05 attention of nsa_attention.cu over
//                    those blocks (one KV tile of l' keys per listed block):
//                    pass A exact max / sum per row and softmax_lse, pass B
//                    P = 2^(s*scale*log2e - m - log2 L) into tensor memory and
//                    O += P V; a row masks the columns of a block it did not
//                    list, and the causal / sequence-end columns.
// Warp roles as in nsa_attention.cu (384 threads): warps 0-3 softmax, warps
// 4-7 epilogue (O read-out), warp 8 TMA producer, warp 9 MMA issuer (and
// tensor-memory owner), warps 10-11 idle.  Every mbarrier wait is bounded; a
// timeout sets the workspace error word and every role drains.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "nsa_internal.h"
#include "ptx.cuh"

namespace nsa {
namespace sel {

enum BarId {
    B_Q_FULL0 = 0,                    // + Q buffer (2)
    B_Q_EMPTY0 = B_Q_FULL0 + 2,       // + Q buffer (2)
    B_S_FULL0 = B_Q_EMPTY0 + 2,       // + score buffer (2)
    B_S_EMPTY0 = B_S_FULL0 + 2,       // + score buffer (2)
    B_P_FULL = B_S_EMPTY0 + 2,
    B_P_EMPTY,
    B_O_FULL,
    B_O_EMPTY,
    B_MMA_DONE,
    B_SLOT_FULL0,                     // + slot (8)
    B_SLOT_EMPTY0 = B_SLOT_FULL0 + 8,
    B_COUNT = B_SLOT_EMPTY0 + 8
};

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
// ---------------------------------------------------------------------------
template <typename T, int LP>
__global__ void __launch_bounds__(kThreads, 1)
sel_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const Params p) {
    constexpr int NKV = LP;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;

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
            mbar_init(bar(B_S_FULL0 + i), 1);
            mbar_init(bar(B_S_EMPTY0 + i), 4);
        }
        mbar_init(bar(B_P_FULL), 4);
        mbar_init(bar(B_P_EMPTY), 1);
        mbar_init(bar(B_O_FULL), 1);
        mbar_init(bar(B_O_EMPTY), 4);
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
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + p.tm_o;
    const uint32_t tmem_p = tmem + p.tm_p;

    const uint32_t q_addr0 = smem_u32(smem + p.off_q);
    const uint32_t ring_addr = smem_u32(smem + p.off_ring);
    const int nslot = p.nslot;
    const int nqbuf = p.nqbuf;
    const int nsbuf = p.nsbuf;
    const int nqc = (p.d1 + 63) / 64;    // 64-element chunks of a Q/K row
    const int nvc = (p.d2 + 63) / 64;    // 64-element chunks of a V row
    // the block list of tile `tile` (written by sel_plan_kernel)
    auto list_n = [&](int tile) { return min(p.list_n[tile], p.cap); };
    auto list_blk = [&](int tile, int i) { return p.list_blk[(size_t)tile * p.cap + i]; };

    if (warp >= 8) setmaxnreg_dec<kRegsCtl>();
    if (warp == 8) {
        // ============================ TMA producer ============================
        // per tile: Q; pass A: K of the listed blocks; pass B: K_0, then
        // K_{i+1}, V_i for each i
        if (lane == 0) {
            uint32_t item = 0;
            int tcount = 0;
            const uint32_t q_bytes = (uint32_t)(nqc * 64 * G * TT * 2);
            const uint32_t k_bytes = (uint32_t)(nqc * 64 * NKV * 2);
            const uint32_t v_bytes = (uint32_t)(nvc * 64 * NKV * 2);
            bool ok = true;
            auto load_kv = [&](bool is_v, int g, int row) {
                const int slot = item % nslot;
                const uint32_t ph = (item / nslot) & 1;
                ok = ok && mbar_wait(bar(B_SLOT_EMPTY0 + slot), ph ^ 1, abort_flag, p.err, kErrTimeoutBase + 2);
                if (!ok) return;
                const uint32_t fb = bar(B_SLOT_FULL0 + slot);
                const uint32_t dst = ring_addr + slot * p.slot_bytes;
                mbar_arrive_expect_tx(fb, is_v ? v_bytes : k_bytes);
                const int nc = is_v ? nvc : nqc;
                for (int c = 0; c < nc; ++c)
                    tma_load_3d(dst + c * NKV * 128, is_v ? &tm_v : &tm_k, c * 64, g, row, fb);
                ++item;
            };
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tcount) {
                const Tile t = p.tiles[tile];
                const int n = list_n(tile);
                const int qb = tcount % nqbuf;
                const uint32_t qph = (tcount / nqbuf) & 1;
                ok = mbar_wait(bar(B_Q_EMPTY0 + qb), qph ^ 1, abort_flag, p.err, kErrTimeoutBase + 3);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(B_Q_FULL0 + qb), q_bytes);
                const uint32_t qdst = q_addr0 + qb * p.q_bytes;
                for (int c = 0; c < nqc; ++c)
                    tma_load_3d(qdst + c * 16384, &tm_q, c * 64, t.group * G, t.q_row0, bar(B_Q_FULL0 + qb));
                auto row_of = [&](int i) { return t.kv_row0 + list_blk(tile, i) * NKV; };
                for (int i = 0; i < n && ok; ++i) load_kv(false, t.group, row_of(i));
                if (n > 0 && ok) load_kv(false, t.group, row_of(0));
                for (int i = 0; i < n && ok; ++i) {
                    if (i + 1 < n) load_kv(false, t.group, row_of(i + 1));
                    load_kv(true, t.group, row_of(i));
                }
            }
        }
    } else if (warp == 9) {
        // ============================ MMA issuer =============================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_f16(kBF16, 128, NKV, false, false);
            const uint32_t idesc_pv = idesc_f16(kBF16, 128, p.d2, false, true);
            const int nks_qk = p.d1 / 16;
            constexpr int nks_pv = NKV / 16;
            uint32_t item = 0, scnt = 0, pcnt = 0;
            int tcount = 0;
            bool ok = true;
            uint32_t q_addr = q_addr0;
            auto issue_s = [&]() {
                const int sb = scnt % nsbuf;
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
                    const uint64_t ad = sdesc_sw128(q_addr + (ks >> 2) * 16384 + off, 16, 1024);
                    const uint64_t bd = sdesc_sw128(kbase + (ks >> 2) * (NKV * 128) + off, 16, 1024);
                    umma_ss(tmem + sb * 128, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
                }
                umma_commit(bar(B_S_FULL0 + sb));
                umma_commit(bar(B_SLOT_EMPTY0 + slot));
                ++item;
                ++scnt;
            };
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tcount) {
                const int n = list_n(tile);
                const int qb = tcount % nqbuf;
                ok = mbar_wait(bar(B_Q_FULL0 + qb), (tcount / nqbuf) & 1, abort_flag, p.err, kErrTimeoutBase + 6);
                if (!ok) break;
                tc_fence_after();
                q_addr = q_addr0 + qb * p.q_bytes;
                for (int i = 0; i < n && ok; ++i) issue_s();          // pass A
                if (n > 0 && ok) issue_s();                          // pass B, S_0
                for (int i = 0; i < n && ok; ++i) {
                    if (i + 1 < n) issue_s();
                    if (i == 0)
                        ok = ok && mbar_wait(bar(B_O_EMPTY), (tcount & 1) ^ 1, abort_flag, p.err,
                                             kErrTimeoutBase + 7);
                    ok = ok && mbar_wait(bar(B_P_FULL), pcnt & 1, abort_flag, p.err, kErrTimeoutBase + 8);
                    const int slot = item % nslot;
                    ok = ok && mbar_wait(bar(B_SLOT_FULL0 + slot), (item / nslot) & 1, abort_flag, p.err,
                                         kErrTimeoutBase + 9);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t vbase = ring_addr + slot * p.slot_bytes;
#pragma unroll
                    for (int ks = 0; ks < nks_pv; ++ks) {
                        const uint64_t bd = sdesc_sw128(vbase + ks * 2048, NKV * 128, 1024);
                        umma_ts(tmem_o, tmem_p + ks * 8, bd, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(bar(B_P_EMPTY));
                    umma_commit(bar(B_SLOT_EMPTY0 + slot));
                    ++item;
                    ++pcnt;
                }
                if (!ok) break;
                // a tile without P V work waits for the previous read-out, so that
                // O_FULL never runs two phases ahead of its consumer
                if (n == 0)
                    ok = mbar_wait(bar(B_O_EMPTY), (tcount & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 7);
                if (!ok) break;
                umma_commit(bar(B_O_FULL));
                umma_commit(bar(B_Q_EMPTY0 + qb));
            }
            // every MMA issued so far has retired before the tensor memory is freed
            umma_commit(bar(B_MMA_DONE));
            mbar_wait(bar(B_MMA_DONE), 0, abort_flag, nullptr, 0);
        }
    } else if (warp < 4) {
        // ===================== softmax (128 thr) =====================
        setmaxnreg_inc<kRegsSoftmax>();
        const int row = warp * 32 + lane;          // tile row = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float c2 = p.scale_log2;
        const int h = row % G;
        const int tok = row / G;
        uint32_t scnt = 0, pcnt = 0;

        auto load_s = [&](float (&s)[NKV]) {
            const int sb = scnt % nsbuf;
            mbar_wait(bar(B_S_FULL0 + sb), (scnt / nsbuf) & 1, abort_flag, p.err, kErrTimeoutBase + 10);
            tc_fence_after();
            const uint32_t ta = tmem + lane_off + sb * 128;
#pragma unroll
            for (int c = 0; c < NKV / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(ta + c * 32, r);
#pragma unroll
                for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[e]);
            }
            if constexpr (NKV % 32 != 0) {
                uint32_t r[16];
                tmem_ld16(ta + (NKV / 32) * 32, r);
#pragma unroll
                for (int e = 0; e < 16; ++e) s[(NKV / 32) * 32 + e] = __uint_as_float(r[e]);
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_S_EMPTY0 + sb));
            ++scnt;
        };
        // scores in "exponent units": x = s * ce - shift.  With a positive scale
        // the raw scores are used as they are (ce = c2); a zero or negative
        // scale first multiplies them in (ce = 1).  Columns c >= lim are not
        // attended to and become -inf.
        const bool pos_scale = c2 > 0.f;
        const float ce = pos_scale ? c2 : 1.f;
        auto prep = [&](float (&s)[NKV], int lim) {
            if (!pos_scale) {
#pragma unroll
                for (int c = 0; c < NKV; ++c) s[c] *= c2;
            }
            if (lim < NKV) {
#pragma unroll
                for (int c = 0; c < NKV; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
            }
        };

        int tcount = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
            const Tile t = p.tiles[tile];
            const int n = list_n(tile);
            const bool valid = (row < TT * G) && (tok < t.ntok);
            const int tpos = t.t0 + tok;
            // columns of listed block i this row attends to: a prefix, cut by the
            // causal rule and the end of the sequence; none when its token did
            // not list the block
            auto lim_of = [&](int i) {
                if (!valid) return 0;
                const int b = list_blk(tile, i);
                const uint32_t w = p.list_mask[((size_t)tile * p.cap + i) * 4 + (tok >> 5)];
                if (!((w >> (tok & 31)) & 1u)) return 0;
                const int lim = min(NKV, min(tpos - b * NKV + 1, t.s_kv - b * NKV));
                return lim > 0 ? lim : 0;
            };

            // ---------------- pass A: exact row max and sum (log2 domain) ----------------
            float m = -INFINITY, L = 0.f;
            for (int i = 0; i < n; ++i) {
                float s[NKV];
                const int lim = lim_of(i);
                load_s(s);
                prep(s, lim);
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < NKV; c += 8) {
                    mx4[0] = fmax3(mx4[0], s[c + 0], s[c + 1]);
                    mx4[1] = fmax3(mx4[1], s[c + 2], s[c + 3]);
                    mx4[2] = fmax3(mx4[2], s[c + 4], s[c + 5]);
                    mx4[3] = fmax3(mx4[3], s[c + 6], s[c + 7]);
                }
                const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * ce;
                const float mn = fmaxf(m, mx);
                const float mref = (mn == -INFINITY) ? 0.f : mn;
                const float2 ce2 = make_float2(ce, ce), nm2 = make_float2(-mref, -mref);
                float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                 make_float2(0.f, 0.f)};
#pragma unroll
                for (int c = 0; c < NKV; c += 2) {
                    const float2 x = ffma2(make_float2(s[c], s[c + 1]), ce2, nm2);
                    acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], make_float2(ex2(x.x), ex2(x.y)));
                }
                const float2 t01 = fadd2(acc[0], acc[1]), t23 = fadd2(acc[2], acc[3]);
                const float sum = (t01.x + t01.y) + (t23.x + t23.y);
                L = L * ex2(m - mref) + sum;
                m = mn;
            }
            if (valid) {
                // natural log-sum-exp: (m + log2 L) * ln 2
                p.lse[(size_t)(t.q_row0 + tok) * p.n1 + (size_t)t.group * G + h] =
                    (L > 0.f) ? (m + lg2(L)) * 0.69314718055994530942f : -INFINITY;
            }

            // ------------- pass B: P -> TMEM -------------
            // P = 2^(s*c2 - m - log2 L): normalised in the exponent
            const float mb = (L > 0.f) ? m + lg2(L) : INFINITY;
            const float2 ce2b = make_float2(ce, ce), nb2 = make_float2(-mb, -mb);
            for (int i = 0; i < n; ++i) {
                float s[NKV];
                const int lim = lim_of(i);
                load_s(s);
                prep(s, lim);
#pragma unroll
                for (int c = 0; c < NKV; c += 2) {
                    const float2 x = ffma2(make_float2(s[c], s[c + 1]), ce2b, nb2);
                    s[c] = ex2(x.x);
                    s[c + 1] = ex2(x.y);
                }
                // P in the storage dtype -> tensor memory (A operand of P V)
                mbar_wait(bar(B_P_EMPTY), (pcnt & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 11);
                tc_fence_after();
                if constexpr ((NKV / 2) % 16 == 0) {
#pragma unroll
                    for (int c = 0; c < NKV / 32; ++c) {
                        uint32_t w[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) w[e] = pack2<T>(s[c * 32 + 2 * e], s[c * 32 + 2 * e + 1]);
                        tmem_st16(tmem_p + lane_off + c * 16, w);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < NKV / 16; ++c) {
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) w[e] = pack2<T>(s[c * 16 + 2 * e], s[c * 16 + 2 * e + 1]);
                        tmem_st8(tmem_p + lane_off + c * 8, w);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_P_FULL));
                ++pcnt;
            }
        }
    } else if (warp < 8) {
        // ============ epilogue: O read-out (128 thr) ============
        setmaxnreg_dec<kRegsEpilogue>();
        const int ew = warp - 4;                   // TMEM lane quadrant
        const int erow = ew * 32 + lane;
        const uint32_t lane_off = (uint32_t)(ew * 32) << 16;
        const int eh = erow % G;
        const int etok = erow / G;
        int tcount = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
            const Tile t = p.tiles[tile];
            const int n = list_n(tile);
            mbar_wait(bar(B_O_FULL), tcount & 1, abort_flag, p.err, kErrTimeoutBase + 12);
            tc_fence_after();
            const bool valid = (erow < TT * G) && (etok < t.ntok);
            T* orow = reinterpret_cast<T*>(p.out) +
                      ((size_t)(t.q_row0 + etok) * p.n1 + (size_t)t.group * G + eh) * p.d2;
            // a row whose token attends to nothing has P = 0 everywhere, so O = 0
            // from the P V products; a tile with no listed block has no P V
            for (int c = 0; c < p.d2 / 16; ++c) {
                uint32_t r[16];
                tmem_ld16(tmem_o + lane_off + c * 16, r);
                tmem_wait_ld();
                if (valid) {
                    uint4 w0, w1;
                    float f[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) f[q] = (n > 0) ? __uint_as_float(r[q]) : 0.f;
                    w0.x = pack2<T>(f[0], f[1]);
                    w0.y = pack2<T>(f[2], f[3]);
                    w0.z = pack2<T>(f[4], f[5]);
                    w0.w = pack2<T>(f[6], f[7]);
                    w1.x = pack2<T>(f[8], f[9]);
                    w1.y = pack2<T>(f[10], f[11]);
                    w1.z = pack2<T>(f[12], f[13]);
                    w1.w = pack2<T>(f[14], f[15]);
                    *reinterpret_cast<uint4*>(orow + c * 16) = w0;
                    *reinterpret_cast<uint4*>(orow + c * 16 + 8) = w1;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_O_EMPTY));
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
    if (warp == 9) {
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
    kern<<<grid, kThreads, p.smem_bytes, st>>>(tq, tk, tv, p);
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
