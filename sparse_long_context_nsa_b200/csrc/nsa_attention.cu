// nsa_attention.cu -- fused compressed attention + importance + top-k (sm_100a),
// two CTAs per SM.
//
// "mindspore.ops.nsa_compress_attention", description steps 1-7:
//   1  S = scale * q . kcmp^T over the visible compressed blocks
//   2  P = softmax(S)
//   3  out = P . vcmp
//   4  P_slc[j] = sum_{m<a} sum_{n<b} P[a*j - m - n],  a = l'/d, b = l/d
//   5  P_slc' = sum over the query heads of one KV group
//   7  top-k of P_slc' over the causal candidates of the query
//
// One M-tile = 128 rows = (128/G consecutive tokens) x (the G query heads of
// one KV group): every row of a tile shares one K/V head, and the group sum of
// step 5 is a sum over neighbouring rows.  Two passes over the compressed
// keys, because step 5 adds *normalised* probabilities of different heads and
// a head's normaliser is only known at the end of its row:
//   pass A  S = Q K^T (tcgen05.mma, operands in shared memory, fp32 in tensor
//           memory); online max / sum in registers -> exact m and L per row;
//           softmax_max / softmax_sum are written here.
//   pass B  S = Q K^T again; P = 2^(s*scale*log2e - m - log2 L) in fp32
//           registers; P (storage dtype) is written back over the first NKV/2
//           score columns and O += P V reads it from there as the A operand;
//           from the fp32 P the banded sum of step 4 goes to a shared-memory
//           staging ring.  At the end of the tile the same warps read O out.
//   epilogue  staged band values summed over the G rows of each token into a
//           per-token score buffer (step 5); top-k (step 7).
// Warp roles (256 threads): warps 0-3 softmax (warp w owns TMEM lanes
// 32w..32w+31 = tile rows), warp 4 TMA producer, warp 5 MMA issuer (and
// tensor-memory owner), warps 6-7 epilogue.  Within one CTA the tile is a
// chain (S, softmax, P V, next S); two CTAs share each SM (about 110 KB of
// shared memory and 256 tensor-memory columns each), so one CTA's
// exponentials run while the other's MMAs and copies are in flight.  Value
// dims above 128 take 512 columns and one CTA per SM.
// Tensor memory: scores at [0, NKV), O from column 128.  Q, K and V are
// staged by TMA with 128-byte swizzle; K and V share one ring, loaded and
// consumed in one fixed order.
// Every mbarrier wait is bounded; a timeout sets the workspace error word and
// every role drains without hanging.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "nsa_internal.h"
#include "ptx.cuh"

namespace nsa {

__host__ __device__ constexpr int kv_cols_for(int a) {
    // largest multiple of lcm(16, a) not above 128: every KV tile then holds a
    // whole number of importance anchors (the anchor of selection block j is
    // compressed block a*j)
    return (a == 1 || a == 2 || a == 4 || a == 8) ? 128
           : (a == 3 || a == 6)                   ? 96
           : (a == 5)                             ? 80
                                                  : 112;
}

__host__ __device__ constexpr int chunk_cols_for(int a) {
    // softmax chunk: a multiple of 16 columns (tensor-memory load shapes) and
    // of a (whole anchors), eight anchors or more
    return (a == 1 || a == 2 || a == 4) ? 32 : (a == 3 || a == 6) ? 48 : (a == 8) ? 64 : (a == 5) ? 80 : 112;
}

enum BarId {
    B_Q_FULL0 = 0,                    // + Q buffer (2)
    B_Q_EMPTY0 = B_Q_FULL0 + 2,       // + Q buffer (2)
    B_S_FULL0 = B_Q_EMPTY0 + 2,                        // + score buffer (2)
    B_S_EMPTY0 = B_S_FULL0 + 2,       // + score buffer (2)
    B_P_FULL0 = B_S_EMPTY0 + 2,       // + score buffer (2)
    B_O_FULL = B_P_FULL0 + 2,
    B_O_EMPTY,
    B_STG_FULL0,                      // + slot (2)
    B_STG_EMPTY0 = B_STG_FULL0 + 2,   // + slot (2)
    B_SC_FULL0 = B_STG_EMPTY0 + 2,    // + score buffer (2)
    B_SC_EMPTY0 = B_SC_FULL0 + 2,     // + score buffer (2)
    B_MMA_DONE = B_SC_EMPTY0 + 2,
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

__device__ __forceinline__ int nvis_of(int t, int l, int d, int n_cmp) {
    // compressed block i is visible to position t iff i*d + l - 1 <= t
    if (t < l - 1) return 0;
    return min(n_cmp, (t - l + 1) / d + 1);
}

// Top-k of one token's group scores (step 7), one warp.  Candidates are
// j < ncand; scores for j >= jcov are 0 (no visible block reaches them).
// Scores are >= 0, so their fp32 bit patterns order like the values: the
// k-th largest key is found by a bitwise search from the top bit down (it
// stops early once exactly k keys lie at or above the trial value, which
// then fixes the selected set), and an ordered ballot scan keeps every key
// above it plus the earliest ties, listing the indices in ascending order.
//
// Memory variant: long candidate lists, or more survivors than the filter
// variant's scratch holds.
__device__ __noinline__ void topk_mem(const float* sc, int ncand, int lim, int k, int count, int32_t* dst,
                                      int lane) {
    uint32_t thr = 0;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t trial = thr | (1u << bit);
        int c = 0;
        for (int j = lane; j < lim; j += 32) c += __float_as_uint(sc[j]) >= trial ? 1 : 0;
        c = __reduce_add_sync(0xffffffffu, c);
        if (c >= k) {
            thr = trial;
            if (c == k) break;
        }
    }
    int ngt = 0;
    for (int j = lane; j < lim; j += 32) ngt += __float_as_uint(sc[j]) > thr ? 1 : 0;
    ngt = __reduce_add_sync(0xffffffffu, ngt);
    const int need_eq = k - ngt;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int eq_seen = 0, written = 0;
    for (int base = 0; base < ncand && written < k; base += 32) {
        const int j = base + lane;
        const bool in = j < ncand;
        const uint32_t kv = (j < lim) ? __float_as_uint(sc[j]) : 0u;
        const bool gt = in && kv > thr;
        const bool eq = in && kv == thr;
        const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
        const bool sel = gt || (eq && (eq_seen + __popc(eqm & lt_mask)) < need_eq);
        eq_seen += __popc(eqm);
        const uint32_t selm = __ballot_sync(0xffffffffu, sel);
        if (sel) dst[written + __popc(selm & lt_mask)] = j;
        written += __popc(selm);
    }
    for (int j = written + lane; j < count; j += 32) dst[j] = -1;
}

// Bitonic sort of one value per lane, descending across the warp.
__device__ __forceinline__ uint32_t warp_sort_desc(uint32_t v, int lane) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
        const bool desc = (lane & size) == 0 || size == 32;
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint32_t o = __shfl_xor_sync(0xffffffffu, v, stride);
            const bool lower = (lane & stride) == 0;
            v = (lower == desc) ? max(v, o) : min(v, o);
        }
    }
    return v;
}

// Filter + rank variant.  Keys become u = bits + 1 inside the candidate range
// (u >= 1) and 0 outside it.  With m1 >= m2 the two largest keys of a lane,
// T = max(k-th largest m1, ceil(k/2)-th largest m2) leaves at least k keys at
// or above T, so every key of the top k is among the survivors u >= T (a key
// below T is strictly below the k-th largest and cannot tie with it).  The
// survivors are compacted in index order into `scr` (u then j, kTopkCap each)
// and each one's rank is counted against all others (larger u first, equal u
// by index), which is a strict order; ranks below k are the result.  Returns
// false, writing nothing, when more than kTopkCap keys survive.
template <int NR>
__device__ __forceinline__ bool topk_filter(const float* sc, int ncand, int lim, int k, int count,
                                            int32_t* dst, int lane, uint32_t* scr) {
    // up to 8 keys a lane stay in registers; longer lists are read twice
    constexpr bool kKeep = NR <= 8;
    constexpr int NK = kKeep ? NR : 1;
    uint32_t kept[NK];
    auto ukey = [&](int i) -> uint32_t {
        const int j = lane + 32 * i;
        return (j < lim) ? __float_as_uint(sc[j]) + 1u : (j < ncand ? 1u : 0u);
    };
    uint32_t m1 = 0, m2 = 0;
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const uint32_t x = ukey(i);
        if constexpr (kKeep) kept[i] = x;
        const uint32_t lo = min(m1, x);
        m1 = max(m1, x);
        m2 = max(m2, lo);
    }
    auto key = [&](int i) -> uint32_t {
        if constexpr (kKeep) return kept[i];
        else return ukey(i);
    };
    m1 = warp_sort_desc(m1, lane);
    m2 = warp_sort_desc(m2, lane);
    const uint32_t thr = max(__shfl_sync(0xffffffffu, m1, k - 1), __shfl_sync(0xffffffffu, m2, (k + 1) / 2 - 1));
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t* su = scr;
    uint32_t* sj = scr + kTopkCap;
    int ns = 0;
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const uint32_t x = key(i);
        const bool sv = x >= thr;
        const uint32_t m = __ballot_sync(0xffffffffu, sv);
        const int pos = ns + __popc(m & lt_mask);
        if (sv && pos < kTopkCap) {
            su[pos] = x;
            sj[pos] = (uint32_t)(lane + 32 * i);
        }
        ns += __popc(m);
    }
    if (ns > kTopkCap) return false;
    __syncwarp();
    int written = 0;
#pragma unroll
    for (int r = 0; r < kTopkCap / 32; ++r) {
        if (32 * r < ns) {
            const int pidx = 32 * r + lane;
            const bool in = pidx < ns;
            const uint32_t up = in ? su[pidx] : 0u;
            int rank = 0;
            for (int q = 0; q < ns; ++q) {
                const uint32_t uq = su[q];
                rank += (uq > up || (uq == up && q < pidx)) ? 1 : 0;
            }
            const bool sel = in && rank < k;
            const uint32_t m = __ballot_sync(0xffffffffu, sel);
            if (sel) dst[written + __popc(m & lt_mask)] = (int32_t)sj[pidx];
            written += __popc(m);
        }
    }
    for (int j = written + lane; j < count; j += 32) dst[j] = -1;
    __syncwarp();   // scratch reads done before the next call overwrites it
    return true;
}

__device__ __forceinline__ void warp_topk(const float* sc, int ncand, int jcov, int count,
                                          int32_t* dst, int lane, uint32_t* scr) {
    const int k = min(count, ncand);
    if (k == ncand) {
        for (int j = lane; j < count; j += 32) dst[j] = (j < ncand) ? j : -1;
        return;
    }
    const int lim = min(ncand, jcov);          // keys at j >= lim are 0
    bool done;
    if (ncand <= 8 * 32)
        done = topk_filter<8>(sc, ncand, lim, k, count, dst, lane, scr);
    else if (ncand <= 16 * 32)
        done = topk_filter<16>(sc, ncand, lim, k, count, dst, lane, scr);
    else if (ncand <= 32 * 32)
        done = topk_filter<32>(sc, ncand, lim, k, count, dst, lane, scr);
    else
        done = false;
    // many ties at the threshold, or a very long candidate list
    if (!done) topk_mem(sc, ncand, lim, k, count, dst, lane);
}

template <typename T, int A>
__global__ void __launch_bounds__(kAttnThreads, 2)
nsa_cmp_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    constexpr int NKV = kv_cols_for(A);            // compressed blocks per KV tile
    constexpr int NJ = NKV / A;                    // importance anchors per KV tile
    constexpr int NTAP = 2 * A - 1;                // band taps u = 0 .. 2A-2 (b <= a)
    constexpr int NCARRY = (2 * A - 2) > 0 ? (2 * A - 2) : 1;
    constexpr int ENT = NJ < kEntryMax ? NJ : kEntryMax;   // anchors per staging entry
    constexpr int NENT = NJ / ENT;                 // staging entries per KV tile
    constexpr int STR = ENT + 4;                   // staging row stride in floats
    constexpr int CW = chunk_cols_for(A);          // score columns per softmax chunk
    constexpr int NC = NKV / CW;                   // chunks per KV tile
    constexpr int NA = CW / A;                     // anchors per chunk
    constexpr int EPC = NA / ENT;                  // staging entries (or group sums) per chunk
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    static_assert(NJ % ENT == 0 && ENT % 4 == 0, "anchor chunking");
    static_assert(NKV % CW == 0 && CW % A == 0 && NA % ENT == 0 && NC * EPC == NENT, "chunk layout");

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
    // tiles of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int nt = (p.num_tiles > (int)blockIdx.x) ? (p.num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto tile_of = [&](int j) { return p.tiles[blockIdx.x + (size_t)j * gridDim.x]; };

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(B_Q_FULL0 + i), 1);
            mbar_init(bar(B_Q_EMPTY0 + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(B_S_FULL0 + i), 1);
            mbar_init(bar(B_S_EMPTY0 + i), 4);
            mbar_init(bar(B_P_FULL0 + i), 4);
        }
        mbar_init(bar(B_O_FULL), 1);
        mbar_init(bar(B_O_EMPTY), 4);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(B_STG_FULL0 + i), 4);
            mbar_init(bar(B_STG_EMPTY0 + i), kEpiWarps);
            mbar_init(bar(B_SC_FULL0 + i), 4);
            mbar_init(bar(B_SC_EMPTY0 + i), kEpiWarps);
        }
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
        tmem_alloc(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // score buffers 128 columns apart (P in the storage dtype over the first
    // NKV/2 columns of the buffer it came from), then the output accumulator
    // (D2 columns).  S tile s uses buffer s % SB, for the (s / SB)-th time.
    const int SB = p.sbufs;
    const uint32_t tmem_s = tmem;
    const uint32_t tmem_o = tmem + SB * 128;
    auto sbuf_of = [&](uint32_t sidx) { return SB == 2 ? (int)(sidx & 1) : 0; };
    auto suse_of = [&](uint32_t sidx) { return SB == 2 ? (sidx >> 1) : sidx; };

    // Q of tile j in buffer j % QB, used for the (j / QB)-th time
    const int QB = p.qbufs;
    auto qbuf_of = [&](int j) { return QB == 2 ? (j & 1) : 0; };
    auto quse_of = [&](int j) { return QB == 2 ? (j >> 1) : j; };
    auto q_addr_of = [&](int j) { return smem_u32(smem + p.off_q) + (uint32_t)(qbuf_of(j) * p.q_bytes); };
    const uint32_t ring_addr = smem_u32(smem + p.off_ring);
    const int nslot = p.nslot;
    const int nqc = (p.d1 + 63) / 64;    // 64-element chunks of a Q/K row
    const int nvc = (p.d2 + 63) / 64;    // 64-element chunks of a V row

    if (warp >= 4) {
        setmaxnreg_to<kRegsSide, kRegsLaunch>();
        if (warp == kWarpTma && lane == 0) {
            // ============================ TMA producer ============================
            // per tile: Q; pass A: K_0..K_{n-1}; pass B: the keys run SB tiles
            // ahead of the values: K_0 .. K_{SB-1}, then V_i, K_{i+SB} for each i
            uint32_t item = 0;
            const uint32_t q_bytes = (uint32_t)(nqc * 64 * G * TT * 2);
            const uint32_t k_bytes = (uint32_t)(nqc * 64 * NKV * 2);
            const uint32_t v_bytes = (uint32_t)(nvc * 64 * NKV * 2);
            bool ok = true;
            auto load_kv = [&](bool is_v, int g, int row) {
                const int slot = item % nslot;
                ok = ok && mbar_wait(bar(B_SLOT_EMPTY0 + slot), ((item / nslot) & 1) ^ 1, abort_flag, p.err,
                                     kErrTimeoutBase + 2);
                if (!ok) return;
                const uint32_t fb = bar(B_SLOT_FULL0 + slot);
                const uint32_t dst = ring_addr + slot * p.slot_bytes;
                mbar_arrive_expect_tx(fb, is_v ? v_bytes : k_bytes);
                const int nc = is_v ? nvc : nqc;
                for (int c = 0; c < nc; ++c)
                    tma_load_3d(dst + c * NKV * 128, is_v ? &tm_v : &tm_k, c * 64, g, row, fb);
                ++item;
            };
            for (int j = 0; j < nt && ok; ++j) {
                const AttnTile t = tile_of(j);
                const int qb = qbuf_of(j);
                ok = mbar_wait(bar(B_Q_EMPTY0 + qb), (quse_of(j) & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 3);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(B_Q_FULL0 + qb), q_bytes);
                for (int c = 0; c < nqc; ++c)
                    tma_load_3d(q_addr_of(j) + c * 16384, &tm_q, c * 64, t.group * G, t.q_row0, bar(B_Q_FULL0 + qb));
                for (int i = 0; i < t.nkv && ok; ++i) load_kv(false, t.group, t.cmp_row0 + i * NKV);
                for (int i = 0; i < t.nkv && i < SB && ok; ++i) load_kv(false, t.group, t.cmp_row0 + i * NKV);
                for (int i = 0; i < t.nkv && ok; ++i) {
                    load_kv(true, t.group, t.cmp_row0 + i * NKV);
                    if (i + SB < t.nkv) load_kv(false, t.group, t.cmp_row0 + (i + SB) * NKV);
                }
            }
        } else if (warp == kWarpMma && lane == 0) {
            // ============================ MMA issuer =============================
            constexpr uint32_t idesc_qk = idesc_f16(kBF16, 128, NKV, false, false);
            const uint32_t idesc_pv = idesc_f16(kBF16, 128, p.d2, false, true);
            const int nks_qk = p.d1 / 16;
            constexpr int nks_pv = NKV / 16;
            // P_FULL per score buffer: with two buffers the softmax may finish P
            // of both before the issuer waits for the first, never more
            uint32_t item = 0, scnt = 0, pcnt[2] = {0u, 0u};
            bool ok = true;
            auto wait_full = [&]() {
                const int slot = item % nslot;
                ok = ok && mbar_wait(bar(B_SLOT_FULL0 + slot), (item / nslot) & 1, abort_flag, p.err,
                                     kErrTimeoutBase + 5);
                return slot;
            };
            // S = Q K^T (K tile in ring slot `slot`) into the score buffer of S tile scnt
            uint32_t q_addr = 0;   // Q of the current tile
            auto issue_s = [&](int slot) {
                const int sb = sbuf_of(scnt);
                ok = ok && mbar_wait(bar(B_S_EMPTY0 + sb), (suse_of(scnt) & 1) ^ 1, abort_flag, p.err,
                                     kErrTimeoutBase + 4);
                if (!ok) return;
                tc_fence_after();
                const uint32_t kbase = ring_addr + slot * p.slot_bytes;
                for (int ks = 0; ks < nks_qk; ++ks) {
                    const uint32_t off = (ks & 3) * 32;   // 16 elements inside a 128-byte row
                    const uint64_t ad = sdesc_sw128(q_addr + (ks >> 2) * 16384 + off, 16, 1024);
                    const uint64_t bd = sdesc_sw128(kbase + (ks >> 2) * (NKV * 128) + off, 16, 1024);
                    umma_ss(tmem_s + sb * 128, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
                }
                umma_commit(bar(B_S_FULL0 + sb));
                umma_commit(bar(B_SLOT_EMPTY0 + slot));
                ++scnt;
                ++item;
            };
            for (int j = 0; j < nt && ok; ++j) {
                const int n = tile_of(j).nkv;
                const int qb = qbuf_of(j);
                q_addr = q_addr_of(j);
                ok = mbar_wait(bar(B_Q_FULL0 + qb), quse_of(j) & 1, abort_flag, p.err, kErrTimeoutBase + 6);
                if (!ok) break;
                tc_fence_after();
                for (int i = 0; i < n && ok; ++i) issue_s(wait_full());                  // pass A
                // pass B: S_0 .. S_{SB-1}, then P_i V_i, S_{i+SB} for each i: a score
                // buffer is refilled right after the P V that reads the P written
                // over it (tcgen05.mma from one thread runs in issue order)
                const uint32_t sb0 = scnt;   // S count of pass B's first tile
                for (int i = 0; i < n && i < SB && ok; ++i) issue_s(wait_full());
                if (n > 0 && n <= SB && ok) umma_commit(bar(B_Q_EMPTY0 + qb));   // last read of Q
                for (int i = 0; i < n && ok; ++i) {
                    const int sv = wait_full();
                    if (i == 0)   // O of the previous tile has been read out
                        ok = ok && mbar_wait(bar(B_O_EMPTY), (j & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 7);
                    const int pb = sbuf_of(sb0 + i);
                    ok = ok && mbar_wait(bar(B_P_FULL0 + pb), pcnt[pb] & 1, abort_flag, p.err, kErrTimeoutBase + 8);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t vbase = ring_addr + sv * p.slot_bytes;
                    const uint32_t pbuf = tmem_s + pb * 128;
#pragma unroll
                    for (int ks = 0; ks < nks_pv; ++ks) {
                        const uint64_t bd = sdesc_sw128(vbase + ks * 2048, NKV * 128, 1024);
                        umma_ts(tmem_o, pbuf + ks * 8, bd, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(bar(B_SLOT_EMPTY0 + sv));
                    ++item;
                    ++pcnt[pb];
                    if (i + SB < n) {
                        issue_s(wait_full());
                        if (i + SB + 1 == n && ok) umma_commit(bar(B_Q_EMPTY0 + qb));   // last read of Q
                    }
                }
                if (!ok) break;
                if (n == 0) {
                    // no P V: keep O_FULL one phase behind the previous read-out
                    ok = mbar_wait(bar(B_O_EMPTY), (j & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 7);
                    if (!ok) break;
                    umma_commit(bar(B_Q_EMPTY0 + qb));
                }
                umma_commit(bar(B_O_FULL));
            }
            // every MMA issued so far has retired before the tensor memory is freed
            umma_commit(bar(B_MMA_DONE));
            mbar_wait(bar(B_MMA_DONE), 0, abort_flag, nullptr, 0);
        } else if (warp >= kWarpEpi0) {
            // ======== epilogue (2 warps): top-k of step 7 (and the group sum of ========
            // ======== step 5 when the softmax warps stage band values instead) ========
            const int ew = warp - kWarpEpi0;
            const int et = ew * 32 + lane;             // 0 .. 32 * kEpiWarps - 1
            constexpr int NE = 32 * kEpiWarps;
            const float* stage = reinterpret_cast<const float*>(smem + p.off_stage);
            const int cap = p.score_cap;
            float* score0 = p.score_in_smem ? reinterpret_cast<float*>(smem + p.off_score)
                                            : p.score_gmem + (size_t)blockIdx.x * 2 * TT * cap;
            uint32_t* topk_scr = reinterpret_cast<uint32_t*>(smem + p.off_topk);
            uint32_t stg = 0;
            for (int j = 0; j < nt; ++j) {
                const AttnTile t = tile_of(j);
                const int buf = j & 1;
                float* score = score0 + (size_t)buf * TT * cap;
                if (p.shfl_group) {
                    // the softmax warps wrote the group sums of this tile
                    mbar_wait(bar(B_SC_FULL0 + buf), (j >> 1) & 1, abort_flag, p.err, kErrTimeoutBase + 15);
                } else {
                    // staged band values summed over the G rows of each token
                    const int nent = t.nkv > 0 ? t.nkv * NENT + 1 : 0;
                    for (int e = 0; e < nent; ++e) {
                        const int slot = stg & 1;
                        mbar_wait(bar(B_STG_FULL0 + slot), (stg >> 1) & 1, abort_flag, p.err, kErrTimeoutBase + 14);
                        const int j0 = (e < t.nkv * NENT) ? (e / NENT) * NJ + (e % NENT) * ENT : t.nkv * NJ;
                        const float* st = stage + (size_t)slot * (p.stage_entry_bytes / 4);
                        for (int pi = et; pi < t.ntok * ENT; pi += NE) {
                            const int tau = pi / ENT, jj = pi - tau * ENT;
                            const float* src = st + (tau * G) * STR + jj;
                            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                            int hh = 0;
                            for (; hh + 4 <= G; hh += 4) {
                                a0 += src[(hh + 0) * STR];
                                a1 += src[(hh + 1) * STR];
                                a2 += src[(hh + 2) * STR];
                                a3 += src[(hh + 3) * STR];
                            }
                            for (; hh < G; ++hh) a0 += src[hh * STR];
                            const int jx = j0 + jj;
                            if (jx < cap) score[tau * cap + jx] = (a0 + a1) + (a2 + a3);
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B_STG_EMPTY0 + slot));
                        ++stg;
                    }
                    // every group sum of this tile is in the score buffer; the two
                    // buffers alternate, so the next tile's sums cannot overwrite
                    // one that the other warp still reads
                    named_bar_sync(2, NE);
                }
                const int jcov = t.nkv > 0 ? t.nkv * NJ + ENT : 0;
                for (int tau = ew; tau < t.ntok; tau += kEpiWarps) {
                    const int tp = t.t0 + tau;
                    int32_t* dst = p.topk + ((size_t)(t.q_row0 + tau) * p.n2 + t.group) * p.count;
                    if (nvis_of(tp, p.l, p.d, t.n_cmp) == 0) {
                        for (int q = lane; q < p.count; q += 32) dst[q] = -1;
                    } else {
                        const int ncand = min(t.n_sel, tp / p.lp + 1);
                        warp_topk(score + tau * cap, ncand, jcov, p.count, dst, lane, topk_scr + ew * 2 * kTopkCap);
                    }
                }
                if (p.shfl_group) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(B_SC_EMPTY0 + buf));
                }
            }
        }
    } else {
        // ===================== softmax warpgroup (warps 0-3, 128 thr) =====================
        // Each KV tile is taken in chunks of CW score columns (a whole number of
        // anchors), one chunk in registers while the next one loads, so that
        // the loop body stays small.
        setmaxnreg_to<kRegsSoftmax, kRegsLaunch>();
        const int row = warp * 32 + lane;          // tile row = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t ts = tmem_s + lane_off;
        const float c2 = p.scale_log2;
        const int a = p.a, bb = p.b;
        float wband[NTAP];
#pragma unroll
        for (int u = 0; u < NTAP; ++u) {
            // multiplicity of m + n = u with m < a, n < b (the double sum of step 4)
            const int c = min(min(u, a - 1), min(bb - 1, a + bb - 2 - u)) + 1;
            wband[u] = (u <= a + bb - 2) ? (float)c : 0.f;
        }
        // scores in "exponent units": x = s * ce - shift.  With a positive scale
        // the raw scores are used as they are (ce = c2); a zero or negative
        // scale first multiplies them in (ce = 1).  Columns c >= lim are not
        // visible and become -inf.
        const bool pos_scale = c2 > 0.f;
        const float ce = pos_scale ? c2 : 1.f;
        auto prep = [&](float (&x)[CW], const uint32_t* r, int lim) {
#pragma unroll
            for (int c = 0; c < CW; ++c) x[c] = pos_scale ? __uint_as_float(r[c]) : __uint_as_float(r[c]) * c2;
            if (lim < CW) {
#pragma unroll
                for (int c = 0; c < CW; ++c) x[c] = (c < lim) ? x[c] : -INFINITY;
            }
        };
        uint32_t scnt = 0;
        // S tile `scnt` is in tensor memory: its first chunk starts loading
        uint32_t tsb = ts;   // score buffer of S tile scnt
        int sbuf = 0;
        auto open_s = [&](uint32_t* r) {
            sbuf = sbuf_of(scnt);
            tsb = ts + sbuf * 128;
            mbar_wait(bar(B_S_FULL0 + sbuf), suse_of(scnt) & 1, abort_flag, p.err, kErrTimeoutBase + 10);
            tc_fence_after();
            tmem_ld_cols<CW>(tsb, r);
        };
        // chunk c has landed in r: convert it, start loading chunk c + 1 (or
        // release the score columns after the last one)
        auto next_chunk = [&](float (&x)[CW], uint32_t* r, int c, int lim) {
            tmem_wait_ld_regs<CW>(r);
            prep(x, r, lim);
            if (c + 1 < NC) {
                tmem_ld_cols<CW>(tsb + (c + 1) * CW, r);
            } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_S_EMPTY0 + sbuf));
                ++scnt;
            }
        };
        float* stage = reinterpret_cast<float*>(smem + p.off_stage);
        uint32_t stg = 0;
        // one staging entry: ENT anchors of this row -> shared memory
        auto put_entry = [&](const float* v) {
            const int slot = stg & 1;
            mbar_wait(bar(B_STG_EMPTY0 + slot), ((stg >> 1) & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 13);
            float4* dst = reinterpret_cast<float4*>(stage + (size_t)slot * (p.stage_entry_bytes / 4) + row * STR);
#pragma unroll
            for (int q4 = 0; q4 < ENT / 4; ++q4)
                dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_STG_FULL0 + slot));
            ++stg;
        };
        const int h = row % G;
        const int tok = row / G;
        // Group sum of step 5 inside the warp, for G a power of two up to 32:
        // the G rows of a token are G consecutive lanes.  A butterfly over the
        // lane bits halves the ENT-vector three times (partner G/2, G/4, G/8,
        // keeping the upper half where the lane bit is set) and adds whole
        // values over the remaining bits, so that lane holds the token sums of
        // anchors 4 h0 + 2 h1 + h2 + i, i < nv; the lanes whose remaining bits
        // are 0 write them to the score buffer.
        const int cap = p.score_cap;
        float* score0 = p.score_in_smem ? reinterpret_cast<float*>(smem + p.off_score)
                                        : p.score_gmem + (size_t)blockIdx.x * 2 * TT * cap;
        const int gd0 = G >> 1, gd1 = G >> 2, gd2 = G >> 3;
        const int gh0 = (lane & gd0) ? 1 : 0, gh1 = (lane & gd1) ? 1 : 0, gh2 = (lane & gd2) ? 1 : 0;
        const int gnv = 8 >> ((gd0 ? 1 : 0) + (gd1 ? 1 : 0) + (gd2 ? 1 : 0));
        const bool gwriter = (lane & (G >= 16 ? (G >> 3) - 1 : 0)) == 0;
        const int gabase = 4 * gh0 + 2 * gh1 + gh2;
        static_assert(ENT == 8, "the in-warp group sum splits 8 anchors");
        auto group_write = [&](float (&v)[ENT], float* srow, int j0) {
            if (gd0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float snd = gh0 ? v[i] : v[i + 4];
                    const float kp = gh0 ? v[i + 4] : v[i];
                    v[i] = kp + __shfl_xor_sync(0xffffffffu, snd, gd0);
                }
            }
            if (gd1) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float snd = gh1 ? v[i] : v[i + 2];
                    const float kp = gh1 ? v[i + 2] : v[i];
                    v[i] = kp + __shfl_xor_sync(0xffffffffu, snd, gd1);
                }
            }
            if (gd2) {
                const float snd = gh2 ? v[0] : v[1];
                const float kp = gh2 ? v[1] : v[0];
                v[0] = kp + __shfl_xor_sync(0xffffffffu, snd, gd2);
            }
            if (G >= 16) v[0] += __shfl_xor_sync(0xffffffffu, v[0], G >> 4);
            if (G >= 32) v[0] += __shfl_xor_sync(0xffffffffu, v[0], G >> 5);
            if (gwriter) {
#pragma unroll
                for (int i = 0; i < ENT; ++i) {
                    const int jx = j0 + gabase + i;
                    if (i < gnv && jx < cap) srow[jx] = v[i];
                }
            }
        };

        for (int j = 0; j < nt; ++j) {
            const AttnTile t = tile_of(j);
            const int buf = j & 1;
            float* srow = score0 + ((size_t)buf * TT + (tok < TT ? tok : 0)) * cap;
            if (p.shfl_group)   // the epilogue is done with this buffer's previous tile
                mbar_wait(bar(B_SC_EMPTY0 + buf), ((j >> 1) & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 16);
            const bool valid = (row < TT * G) && (tok < t.ntok);
            const int nvis = valid ? nvis_of(t.t0 + tok, p.l, p.d, t.n_cmp) : 0;
            const size_t qrow = (size_t)t.q_row0 + tok;

            // ---------------- pass A: exact row max and sum (log2 domain) ----------------
            float m = -INFINITY, L = 0.f;
            for (int i = 0; i < t.nkv; ++i) {
                uint32_t r[CW];
                open_s(r);
#pragma unroll 1
                for (int c = 0; c < NC; ++c) {
                    float x[CW];
                    next_chunk(x, r, c, nvis - i * NKV - c * CW);
                    // chunk maximum: four independent chains of 3-input max
                    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int q = 0; q < CW; q += 8) {
                        mx4[0] = fmax3(mx4[0], x[q + 0], x[q + 1]);
                        mx4[1] = fmax3(mx4[1], x[q + 2], x[q + 3]);
                        mx4[2] = fmax3(mx4[2], x[q + 4], x[q + 5]);
                        mx4[3] = fmax3(mx4[3], x[q + 6], x[q + 7]);
                    }
                    const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * ce;
                    const float mn = fmaxf(m, mx);
                    const float mref = (mn == -INFINITY) ? 0.f : mn;
                    // chunk sum of 2^(x - mref): packed exponent arguments, 8 partial sums
                    const float2 ce2 = make_float2(ce, ce), nm2 = make_float2(-mref, -mref);
                    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                     make_float2(0.f, 0.f)};
#pragma unroll
                    for (int q = 0; q < CW; q += 2) {
                        const float2 e = ffma2(make_float2(x[q], x[q + 1]), ce2, nm2);
                        acc[(q >> 1) & 3] = fadd2(acc[(q >> 1) & 3], make_float2(ex2(e.x), ex2(e.y)));
                    }
                    const float2 t01 = fadd2(acc[0], acc[1]), t23 = fadd2(acc[2], acc[3]);
                    const float sum = (t01.x + t01.y) + (t23.x + t23.y);
                    L = L * ex2(m - mref) + sum;
                    m = mn;
                }
            }
            if (valid) {
                const size_t si = (qrow * p.n1 + (size_t)t.group * G + h) * 8;
                const float mo = (m == -INFINITY) ? -INFINITY : m * 0.69314718055994530942f;
                const float4 mv = make_float4(mo, mo, mo, mo);
                const float4 lv = make_float4(L, L, L, L);
                reinterpret_cast<float4*>(p.smax + si)[0] = mv;
                reinterpret_cast<float4*>(p.smax + si)[1] = mv;
                reinterpret_cast<float4*>(p.ssum + si)[0] = lv;
                reinterpret_cast<float4*>(p.ssum + si)[1] = lv;
            }

            // ---- pass B: P -> the score columns (TMEM), band values -> group sums ----
            // P = 2^(s*c2 - m - log2 L): normalised in the exponent
            const float mb = (L > 0.f) ? m + lg2(L) : INFINITY;
            float carry[NCARRY];
#pragma unroll
            for (int k = 0; k < NCARRY; ++k) carry[k] = 0.f;
            for (int i = 0; i < t.nkv; ++i) {
                uint32_t r[CW];
                open_s(r);
#pragma unroll 1
                for (int c = 0; c < NC; ++c) {
                    float x[CW];
                    next_chunk(x, r, c, nvis - i * NKV - c * CW);
                    {
                        const float2 ce2 = make_float2(ce, ce), nb2 = make_float2(-mb, -mb);
#pragma unroll
                        for (int q = 0; q < CW; q += 2) {
                            const float2 e = ffma2(make_float2(x[q], x[q + 1]), ce2, nb2);
                            x[q] = ex2(e.x);
                            x[q + 1] = ex2(e.y);
                        }
                    }
                    // P in the storage dtype over score columns [c CW/2, (c+1) CW/2):
                    // the A operand of P V.  Those columns belong to chunks that
                    // have been read already; the MMA issuer writes the next
                    // scores only after this tile's P V.
                    {
                        uint32_t pw[CW / 2];
#pragma unroll
                        for (int e = 0; e < CW / 2; ++e) pw[e] = pack2<T>(x[2 * e], x[2 * e + 1]);
                        tmem_st_cols<CW / 2>(tsb + c * (CW / 2), pw);
                    }
                    // step 4 on the fp32 P: anchors A*jl of this chunk; taps reach
                    // back into the previous chunk through `carry` (carry[k] = P[c0 - 1 - k])
#pragma unroll
                    for (int e = 0; e < EPC; ++e) {
                        float v[ENT];
#pragma unroll
                        for (int qq = 0; qq < ENT; ++qq) {
                            const int anchor = A * (e * ENT + qq);
                            float acc = 0.f;
#pragma unroll
                            for (int u = 0; u < NTAP; ++u) {
                                const int xi = anchor - u;
                                const float pv = (xi >= 0) ? x[xi >= 0 ? xi : 0] : carry[xi < 0 ? (-xi - 1) : 0];
                                acc = fmaf(wband[u], pv, acc);
                            }
                            v[qq] = acc;
                        }
                        if (p.shfl_group)
                            group_write(v, srow, i * NJ + c * NA + e * ENT);
                        else
                            put_entry(v);
                    }
#pragma unroll
                    for (int k = 0; k < NCARRY; ++k) carry[k] = x[CW - 1 - k];
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_P_FULL0 + sbuf));
            }
            if (t.nkv > 0) {
                // the first anchors past the last KV tile still collect taps from it
                float v[ENT];
#pragma unroll
                for (int qq = 0; qq < ENT; ++qq) {
                    const int anchor = A * qq;
                    float acc = 0.f;
#pragma unroll
                    for (int u = 0; u < NTAP; ++u) {
                        const int xi = anchor - u;
                        if (xi < 0) acc = fmaf(wband[u], carry[-xi - 1 >= 0 ? -xi - 1 : 0], acc);
                    }
                    v[qq] = acc;
                }
                if (p.shfl_group)
                    group_write(v, srow, t.nkv * NJ);
                else
                    put_entry(v);
            }
            if (p.shfl_group) {
                // the group sums of this tile are in the score buffer
                __threadfence_block();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_SC_FULL0 + buf));
            }

            // ---- O (tensor memory) -> attention_out ----
            mbar_wait(bar(B_O_FULL), j & 1, abort_flag, p.err, kErrTimeoutBase + 12);
            tc_fence_after();
            {
                T* orow = reinterpret_cast<T*>(p.out) + (qrow * p.n1 + (size_t)t.group * G + h) * p.d2;
                for (int c = 0; c < p.d2 / 16; ++c) {
                    uint32_t r[16];
                    tmem_ld16(tmem_o + lane_off + c * 16, r);
                    tmem_wait_ld();
                    if (valid) {
                        uint4 w0, w1;
                        float f[16];
#pragma unroll
                        for (int q = 0; q < 16; ++q) f[q] = (nvis > 0) ? __uint_as_float(r[q]) : 0.f;
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
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
    }
}

template <typename T, int A>
static cudaError_t launch_t(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, int grid, cudaStream_t st) {
    auto kern = nsa_cmp_attn_kernel<T, A>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
    if (e != cudaSuccess) return e;
    // all of the unified L1 / shared storage as shared memory: two CTAs of
    // about 110 KB each then fit on one SM
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    kern<<<grid, kAttnThreads, p.smem_bytes, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_a(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, int grid, cudaStream_t st) {
    switch (p.a) {
        case 1: return launch_t<T, 1>(p, tq, tk, tv, grid, st);
        case 2: return launch_t<T, 2>(p, tq, tk, tv, grid, st);
        case 3: return launch_t<T, 3>(p, tq, tk, tv, grid, st);
        case 4: return launch_t<T, 4>(p, tq, tk, tv, grid, st);
        case 5: return launch_t<T, 5>(p, tq, tk, tv, grid, st);
        case 6: return launch_t<T, 6>(p, tq, tk, tv, grid, st);
        case 7: return launch_t<T, 7>(p, tq, tk, tv, grid, st);
        case 8: return launch_t<T, 8>(p, tq, tk, tv, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

int attention_kv_cols(int a) { return kv_cols_for(a); }

cudaError_t launch_attention(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, int grid, cudaStream_t st) {
    return p.dtype == 0 ? launch_a<__nv_bfloat16>(p, tq, tk, tv, grid, st)
                        : launch_a<__half>(p, tq, tk, tv, grid, st);
}

}  // namespace nsa
