// nsa_attention.cu -- fused compressed attention + importance + top-k (sm_100a).
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
// step 5 runs over neighbouring rows.  A work item holds one M-tile, or two
// adjacent M-tiles of the same sequence and group that read the same K/V
// tiles (two "pipelines", one softmax warpgroup each).
//
// One pass over the compressed keys per M-tile, online softmax:
//   S = Q K^T (tcgen05.mma, operands in shared memory, fp32 in tensor memory).
//   The softmax warps read S in chunks of CH columns.  Each row keeps a
//   reference maximum m_ref (log2 units) that moves only when a chunk's
//   maximum exceeds it by more than kRescaleLog2; then the row's sum L, the
//   P values already written for the tile and O are rescaled.  P =
//   2^(s*scale*log2e - m_ref) goes, in the storage dtype, over the score
//   columns it came from and O += P V reads it from there (A operand in
//   tensor memory).  The exact maximum is tracked as well for softmax_max.
//   Step 4 needs the *normalised* P of each head, known only at the end of
//   the row, while step 5 adds heads with different normalisers: so the
//   banded sums of the unnormalised fp32 P (step 4 up to a factor) go, per
//   chunk, to a per-CTA scratch row in global memory (sized to stay in L2),
//   with the chunk's m_ref; the row's final m_ref and L go to shared memory.
// Epilogue warps, concurrently with the next item: O / L -> attention_out;
// for each token, P_slc' = sum over the G heads of 2^(m_ref_chunk - m_ref -
// log2 L) x banded value (steps 4-5) into a per-warp score row, then the
// top-k (step 7).
// Warp roles (512 threads, four warpgroups): warps 0-3 softmax of pipeline
// 0, warps 4-7 softmax of pipeline 1 (warp w owns TMEM lanes 32(w%4).. =
// tile rows), warps 8-11 epilogue (same lane quadrants), warp 12 TMA
// producer, warp 13 MMA issuer (and tensor-memory owner), warps 14-15 idle.
// Registers move to the softmax warpgroups with setmaxnreg.  One persistent
// CTA per SM.  Q, K and V are staged by TMA with 128-byte swizzle; K and V
// share one ring of slots.  Every mbarrier wait is bounded; a timeout sets
// the workspace error word and every role drains without hanging.
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
    // score columns per softmax step: a whole number of anchors, a divisor of
    // the KV tile, loadable from tensor memory in pieces of 32/16/8 columns.
    // Measured on B200: 64-column chunks beat 32-column chunks with the next
    // chunk's load in flight (16K workload 1.17 vs 1.26 ms, 128K 49.1 vs 54.1 ms)
    return (a == 1 || a == 2 || a == 4 || a == 8) ? 64 : 8 * a;
}

int attention_kv_cols(int a) { return kv_cols_for(a); }
int attention_chunk_cols(int a) { return chunk_cols_for(a); }

enum BarId {
    B_Q_FULL0 = 0,
    B_Q_FULL1,
    B_Q_EMPTY0,
    B_Q_EMPTY1,
    B_S_FULL = 4,        // + 2 * pipeline + buffer
    B_P_FULL = 8,        // + pipeline: P of the tile written (4 softmax warps)
    B_P_EMPTY = 10,      // + pipeline: the P V of that pipeline completed
    B_O_FULL = 12,       // + pipeline: last P V of the item completed
    B_O_EMPTY = 14,      // + pipeline: O read out (4 epilogue warps)
    B_ROW_DONE = 16,     // + 2 * pipeline + slot: scratch rows and row statistics written (4 softmax
                         // warps); one per slot, so that it never runs two phases ahead of its waiter
    B_SCR_EMPTY = 20,    // + 2 * pipeline + slot: scratch slot read (4 epilogue warps)
    B_MMA_DONE = 24,
    B_SLOT_FULL0 = 25,   // + ring slot
    B_SLOT_EMPTY0 = B_SLOT_FULL0 + 8,
    B_COUNT = B_SLOT_EMPTY0 + 8
};
static_assert(B_COUNT * 8 + 8 <= 512, "barrier area");

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
template <typename T>
__device__ __forceinline__ float2 unpack2(uint32_t w);
template <>
__device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t w) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w));
}
template <>
__device__ __forceinline__ float2 unpack2<__half>(uint32_t w) {
    return __half22float2(*reinterpret_cast<__half2*>(&w));
}

__device__ __forceinline__ int nvis_of(int t, int l, int d, int n_cmp) {
    // compressed block i is visible to position t iff i*d + l - 1 <= t
    if (t < l - 1) return 0;
    return min(n_cmp, (t - l + 1) / d + 1);
}

// k-th largest key (fp32 bit pattern) of sc[0 .. ncand) held in registers,
// NR keys per lane (key i of a lane belongs to j = lane + 32 i); keys at
// j >= lim are 0.  Bitwise search from the top bit down.
// Bit j of a packed mask row (bit j % 32 of word j / 32; set = removed).
__device__ __forceinline__ bool mask_bit(const uint32_t* row, int j) { return (row[j >> 5] >> (j & 31)) & 1u; }

template <int NR, bool kMask>
__device__ __forceinline__ uint32_t kth_key_regs(const float* sc, int ncand, int lim, int k, int lane,
                                                 const uint32_t* trow) {
    uint32_t key[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const int j = lane + 32 * i;
        bool in = j < lim;
        if constexpr (kMask) in = in && !(trow && mask_bit(trow, j));
        key[i] = in ? __float_as_uint(sc[j]) : 0u;
    }
    uint32_t thr = 0;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t trial = thr | (1u << bit);
        int c0 = 0, c1 = 0;
#pragma unroll
        for (int i = 0; i < NR; i += 2) {
            c0 += key[i] >= trial ? 1 : 0;
            c1 += key[i + 1] >= trial ? 1 : 0;
        }
        const int c = __reduce_add_sync(0xffffffffu, c0 + c1);
        if (c >= k) thr = trial;
        // exactly k keys at or above the trial threshold: they are the top-k
        // (the selection below takes the keys above thr, none of which is equal
        // to a threshold that no key reaches exactly, plus none of the ties)
        if (c == k) break;
    }
    return thr;
}

// Top-k of one token's group scores (step 7), one warp.  Candidates are
// j < ncand; scores for j >= jcov are 0 (no visible block reaches them).
// Exact k-th largest key by a bitwise search over the fp32 bit patterns
// (scores are >= 0, so the bit patterns order like the values), then an
// ordered ballot scan keeps every key above it plus the earliest ties, which
// also lists the indices in ascending order.  With a topk_mask row (kMask,
// bit-packed), candidates whose bit is set are out of the set (step 6).
template <bool kMask>
__device__ __forceinline__ void warp_topk(const float* sc, int ncand, int jcov, int count,
                                          int32_t* dst, int lane, const uint32_t* trow) {
    auto masked = [&](int j) {
        if constexpr (kMask) return trow != nullptr && mask_bit(trow, j);
        return false;
    };
    int n_in = ncand;
    if constexpr (kMask) {
        if (trow) {
            // set bits among the candidates, a word per lane
            int nm = 0;
            for (int w = lane; w * 32 < ncand; w += 32) {
                const int left = ncand - w * 32;
                const uint32_t keep = left >= 32 ? 0xffffffffu : ((1u << left) - 1u);
                nm += __popc(trow[w] & keep);
            }
            n_in = ncand - __reduce_add_sync(0xffffffffu, nm);
        }
    }
    const int k = min(count, n_in);
    if (k == n_in && (!kMask || n_in == ncand)) {
        for (int j = lane; j < count; j += 32) dst[j] = (j < ncand) ? j : -1;
        return;
    }
    const int lim = min(ncand, jcov);          // keys at j >= lim are 0
    uint32_t thr = 0;
    if (k == n_in) {
        thr = 0;                               // every remaining candidate is taken
    } else if (ncand <= 8 * 32) {
        thr = kth_key_regs<8, kMask>(sc, ncand, lim, k, lane, trow);
    } else if (ncand <= 16 * 32) {
        thr = kth_key_regs<16, kMask>(sc, ncand, lim, k, lane, trow);
    } else if (ncand <= 32 * 32) {
        thr = kth_key_regs<32, kMask>(sc, ncand, lim, k, lane, trow);
    } else {
#pragma unroll 1
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t trial = thr | (1u << bit);
            int c = 0;
            for (int j = lane; j < lim; j += 32) c += (!masked(j) && __float_as_uint(sc[j]) >= trial) ? 1 : 0;
            c = __reduce_add_sync(0xffffffffu, c);
            if (c >= k) thr = trial;
            if (c == k) break;   // exactly k keys at or above it: the top-k
        }
    }
    int ngt = 0;
    for (int j = lane; j < lim; j += 32) ngt += (!masked(j) && __float_as_uint(sc[j]) > thr) ? 1 : 0;
    ngt = __reduce_add_sync(0xffffffffu, ngt);
    const int need_eq = k - ngt;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int eq_seen = 0, written = 0;
    for (int base = 0; base < ncand && written < k; base += 32) {
        const int j = base + lane;
        const bool in = j < ncand && !masked(j < ncand ? j : 0);
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


// Multiplies n_cols fp32 columns of this warp's 32 tensor-memory lanes by the
// per-lane factor f, in 16-column pieces.
__device__ __noinline__ void tmem_scale_f32(uint32_t taddr, int n_cols, float f) {
    for (int c = 0; c < n_cols; c += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + c, r);
        tmem_wait_ld_regs<16>(r);
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
        tmem_st16(taddr + c, r);
    }
}

// Multiplies NP columns of packed 16-bit pairs (P in the storage dtype) by f.
template <typename T, int NP>
__device__ __noinline__ void tmem_scale_packed(uint32_t taddr, float f) {
    uint32_t r[NP];
    tmem_ld_n<NP>(taddr, r);
    tmem_wait_ld_regs<NP>(r);
#pragma unroll
    for (int e = 0; e < NP; ++e) {
        const float2 v = unpack2<T>(r[e]);
        r[e] = pack2<T>(v.x * f, v.y * f);
    }
    tmem_st_n<NP>(taddr, r);
}

template <typename T, int A, bool kMask, bool kTwoPass>
__global__ void __launch_bounds__(kAttnThreads, 1)
nsa_cmp_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    constexpr int NKV = kv_cols_for(A);            // compressed blocks per KV tile
    constexpr int CH = chunk_cols_for(A);          // score columns per softmax chunk
    constexpr int NCH = NKV / CH;                  // chunks per KV tile
    constexpr int NJ = NKV / A;                    // importance anchors per KV tile
    constexpr int NJC = CH / A;                    // importance anchors per chunk
    constexpr int NTAP = 2 * A - 1;                // band taps u = 0 .. 2A-2 (b <= a)
    constexpr int NCARRY = (2 * A - 2) > 0 ? (2 * A - 2) : 1;
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr bool kPrefetch = CH <= 32;           // next chunk's load in flight while this one runs
                                                   // (32-column chunks only: registers)
    static_assert(NKV % CH == 0 && CH % A == 0 && NJC % 4 == 0 && CH >= NCARRY, "chunking");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + p.off_bar + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.off_bar + 8 * B_COUNT + 4);
    float* rowstat = reinterpret_cast<float*>(smem + p.off_rowstat);   // [pipe][slot][m_ref, L][128]
    auto bar = [&](int id) { return smem_u32(&bars[id]); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.G;
    const int TT = p.tok_per_tile;
    const int npipe = p.npipe;
    const int nsb = p.nsb;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(bar(B_Q_FULL0 + i), 1);
        for (int i = 0; i < 4; ++i) mbar_init(bar(B_S_FULL + i), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(B_P_FULL + i), 4);
            mbar_init(bar(B_P_EMPTY + i), 1);
            mbar_init(bar(B_O_FULL + i), 1);
            mbar_init(bar(B_O_EMPTY + i), 4);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar(B_ROW_DONE + i), 4);
            mbar_init(bar(B_SCR_EMPTY + i), 4);
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
    if (warp == 13) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const uint32_t q_addr0 = smem_u32(smem + p.off_q);
    const uint32_t ring_addr = smem_u32(smem + p.off_ring);
    const int nslot = p.nslot;
    const int nqbuf = p.nqbuf;
    const int nqc = (p.d1 + 63) / 64;    // 64-element chunks of a Q/K row
    const int nvc = (p.d2 + 63) / 64;    // 64-element chunks of a V row
    const uint32_t q_tile_stride = (uint32_t)nqc * 16384u;   // one M-tile of Q in shared memory

    if (warp >= 12) {
        setmaxnreg_dec<kRegsCtl>();
        if (warp == 12 && lane == 0) {
            // ============================ TMA producer ============================
            uint32_t item = 0;
            int tcount = 0;
            const uint64_t q_policy = l2_policy_evict_first();
            const uint32_t q_bytes = (uint32_t)(nqc * 64 * G * TT * 2);   // one M-tile box
            const uint32_t k_bytes = (uint32_t)(nqc * 64 * NKV * 2);
            const uint32_t v_bytes = (uint32_t)(nvc * 64 * NKV * 2);
            bool ok = true;
            // K or V tile kt of item t: NKV compressed rows from the sequence's contiguous
            // rows, or, with a block table, page by page (an entry past the sequence's pages
            // reads rows beyond the pool, which the copy fills with zeros)
            auto load_kv = [&](bool is_v, const AttnTile& t, int kt) {
                const int g = t.group;
                const int slot = item % nslot;
                const uint32_t ph = (item / nslot) & 1;
                ok = ok && mbar_wait(bar(B_SLOT_EMPTY0 + slot), ph ^ 1, abort_flag, p.err, kErrTimeoutBase + 2);
                if (!ok) return;
                const uint32_t fb = bar(B_SLOT_FULL0 + slot);
                const uint32_t dst = ring_addr + slot * p.slot_bytes;
                mbar_arrive_expect_tx(fb, is_v ? v_bytes : k_bytes);
                const int nc = is_v ? nvc : nqc;
                const CUtensorMap* map = is_v ? &tm_v : &tm_k;
                if (p.block_table == nullptr) {
                    const int row = t.cmp_row0 + kt * NKV;
                    for (int c = 0; c < nc; ++c) tma_load_3d(dst + c * NKV * 128, map, c * 64, g, row, fb);
                } else {
                    const int pr = p.page_rows, npg = (t.n_cmp + pr - 1) / pr;
                    for (int pg = 0; pg < NKV / pr; ++pg) {
                        const int logical = kt * (NKV / pr) + pg;
                        const int row = logical < npg ? p.block_table[(size_t)t.seq * p.bt_stride + logical] * pr
                                                      : p.pool_rows;
                        for (int c = 0; c < nc; ++c)
                            tma_load_3d(dst + c * NKV * 128 + pg * pr * 128, map, c * 64, g, row, fb);
                    }
                }
                ++item;
            };
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tcount) {
                const AttnTile t = p.tiles[tile];
                const int qb = tcount % nqbuf;
                const uint32_t qph = (tcount / nqbuf) & 1;
                ok = mbar_wait(bar(B_Q_EMPTY0 + qb), qph ^ 1, abort_flag, p.err, kErrTimeoutBase + 3);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(B_Q_FULL0 + qb), q_bytes * npipe);
                const uint32_t qdst = q_addr0 + qb * p.q_bytes;
                // Q is read once: evict it first and keep L2 for K/V and the scratch
                for (int pp = 0; pp < npipe; ++pp)
                    for (int c = 0; c < nqc; ++c)
                        tma_load_3d_hint(qdst + pp * q_tile_stride + c * 16384, &tm_q, c * 64, t.group * G,
                                         t.q_row0 + pp * TT, bar(B_Q_FULL0 + qb), q_policy);
                // two passes: first every K tile alone (the row maxima and sums)
                if constexpr (kTwoPass)
                    for (int i = 0; i < t.nkv && ok; ++i) load_kv(false, t, i);
                // K_0, then K_{i+1} ahead of V_i: the order the MMA issuer consumes them
                if (t.nkv > 0 && ok) load_kv(false, t, 0);
                for (int i = 0; i < t.nkv && ok; ++i) {
                    if (i + 1 < t.nkv) load_kv(false, t, i + 1);
                    load_kv(true, t, i);
                }
            }
        } else if (warp == 13 && lane == 0) {
            // ============================ MMA issuer =============================
            constexpr uint32_t idesc_qk = idesc_f16(kBF16, 128, NKV, false, false);
            const uint32_t idesc_pv = idesc_f16(kBF16, 128, p.d2, false, true);
            const int nks_qk = p.d1 / 16;
            constexpr int nks_pv = NKV / 16;
            uint32_t item = 0;
            int scnt0 = 0, scnt1 = 0, pvc0 = 0, pvc1 = 0;   // per pipeline: Q K^T and P V issued
            const uint32_t tm_s0 = tmem + p.tm_s[0], tm_s1 = tmem + p.tm_s[1];
            const uint32_t tm_o0 = tmem + p.tm_o[0], tm_o1 = tmem + p.tm_o[1];
            int tcount = 0;
            bool ok = true;
            auto wait_slot = [&]() {
                const int slot = item % nslot;
                ok = ok && mbar_wait(bar(B_SLOT_FULL0 + slot), (item / nslot) & 1, abort_flag, p.err,
                                     kErrTimeoutBase + 5);
                ++item;
                return slot;
            };
            // S_pp = Q_pp K^T into the next score buffer of pipeline pp
            auto qk = [&](int pp, uint32_t qaddr, int kslot) {
                int& sc = pp ? scnt1 : scnt0;
                const int sb = sc % nsb;
                const uint32_t kbase = ring_addr + kslot * p.slot_bytes;
                const uint32_t qa = qaddr + pp * q_tile_stride;
                const uint32_t dst = (pp ? tm_s1 : tm_s0) + sb * 128;
                for (int ks = 0; ks < nks_qk; ++ks) {
                    const uint32_t off = (ks & 3) * 32;   // 16 elements inside a 128-byte row
                    const uint64_t ad = sdesc_sw128(qa + (ks >> 2) * 16384 + off, 16, 1024);
                    const uint64_t bd = sdesc_sw128(kbase + (ks >> 2) * (NKV * 128) + off, 16, 1024);
                    umma_ss(dst, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
                }
                umma_commit(bar(B_S_FULL + 2 * pp + sb));
                ++sc;
            };
            // O_pp (+)= P_pp V, P read from the score buffer it was written over
            auto pv = [&](int pp, int vslot, bool acc) {
                int& pc = pp ? pvc1 : pvc0;
                ok = ok && mbar_wait(bar(B_P_FULL + pp), pc & 1, abort_flag, p.err, kErrTimeoutBase + 8);
                if (!ok) return;
                tc_fence_after();
                const int sb = pc % nsb;
                const uint32_t vbase = ring_addr + vslot * p.slot_bytes;
                const uint32_t pa = (pp ? tm_s1 : tm_s0) + sb * 128;
                const uint32_t od = pp ? tm_o1 : tm_o0;
#pragma unroll
                for (int ks = 0; ks < nks_pv; ++ks) {
                    const uint64_t bd = sdesc_sw128(vbase + ks * 2048, NKV * 128, 1024);
                    umma_ts(od, pa + ks * 8, bd, idesc_pv, (acc || ks > 0) ? 1u : 0u);
                }
                umma_commit(bar(B_P_EMPTY + pp));
                ++pc;
            };
            for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tcount) {
                const AttnTile t = p.tiles[tile];
                const int qb = tcount % nqbuf;
                ok = mbar_wait(bar(B_Q_FULL0 + qb), (tcount / nqbuf) & 1, abort_flag, p.err, kErrTimeoutBase + 6);
                if (!ok) break;
                tc_fence_after();
                const uint32_t qaddr = q_addr0 + qb * p.q_bytes;
                if constexpr (kTwoPass) {
                    // pass 1: S_i = Q K_i^T for every tile; the softmax reads each S and
                    // hands its buffer back through P_FULL (there is no P V in this pass).
                    // A buffer is reissued only once the S it held has been read.
                    auto consume = [&](int pp) {
                        int& pc = pp ? pvc1 : pvc0;
                        ok = ok && mbar_wait(bar(B_P_FULL + pp), pc & 1, abort_flag, p.err, kErrTimeoutBase + 15);
                        // the softmax's reads of the buffer are ordered before the next MMA into it
                        tc_fence_after();
                        ++pc;
                    };
                    // With two buffers (one pipeline) S_i goes into the buffer that S_{i-2}
                    // left, and the hand-back of S_{i-1} is waited for right after S_i is
                    // issued: nothing may block in between, or the softmax could hand back
                    // two buffers before the first wait and P_FULL would alias a phase.
                    for (int i = 0; i < t.nkv && ok; ++i) {
                        const int ks = wait_slot();
                        if (!ok) break;
                        tc_fence_after();
                        for (int pp = 0; pp < npipe && ok; ++pp) {
                            if (nsb == 1 && i >= 1) consume(pp);
                            if (ok) qk(pp, qaddr, ks);
                        }
                        umma_commit(bar(B_SLOT_EMPTY0 + ks));
                        if (nsb == 2 && i >= 1) consume(0);
                    }
                    if (t.nkv > 0)
                        for (int pp = 0; pp < npipe; ++pp) consume(pp);   // the last S of each pipeline
                    if (!ok) break;
                }
                if (t.nkv > 0) {
                    const int k0 = wait_slot();
                    if (!ok) break;
                    tc_fence_after();
                    for (int pp = 0; pp < npipe; ++pp) qk(pp, qaddr, k0);
                    if (t.nkv == 1) umma_commit(bar(B_Q_EMPTY0 + qb));
                    umma_commit(bar(B_SLOT_EMPTY0 + k0));
                    for (int i = 0; i < t.nkv && ok; ++i) {
                        const int kslot = (i + 1 < t.nkv) ? wait_slot() : -1;
                        const int vslot = wait_slot();
                        if (!ok) break;
                        tc_fence_after();
                        // the epilogue has read the previous item's O out.  Waited for
                        // before S_{i+1} is issued: between that issue and the wait for
                        // P_i nothing may block, or the softmax could finish tiles i and
                        // i+1 first and P_FULL would run two phases ahead of this wait
                        if (i == 0)
                            for (int pp = 0; pp < npipe; ++pp)
                                ok = ok && mbar_wait(bar(B_O_EMPTY + pp), (tcount & 1) ^ 1, abort_flag, p.err,
                                                     kErrTimeoutBase + 7);
                        if (!ok) break;
                        // two score buffers (one pipeline): S_{i+1} goes into the
                        // buffer whose P was consumed by the previous P V
                        if (nsb == 2 && kslot >= 0) qk(0, qaddr, kslot);
                        for (int pp = 0; pp < npipe; ++pp) {
                            pv(pp, vslot, i > 0);
                            // one score buffer: S_{i+1} overwrites P_i after its P V
                            // (tcgen05.mma of one thread execute in issue order)
                            if (nsb == 1 && kslot >= 0 && ok) qk(pp, qaddr, kslot);
                        }
                        if (!ok) break;
                        if (i + 2 == t.nkv) umma_commit(bar(B_Q_EMPTY0 + qb));   // last Q K^T issued
                        umma_commit(bar(B_SLOT_EMPTY0 + vslot));
                        if (kslot >= 0) umma_commit(bar(B_SLOT_EMPTY0 + kslot));
                    }
                } else {
                    // no visible block in the item: keep the O hand-off in step
                    for (int pp = 0; pp < npipe; ++pp)
                        ok = ok && mbar_wait(bar(B_O_EMPTY + pp), (tcount & 1) ^ 1, abort_flag, p.err,
                                             kErrTimeoutBase + 7);
                    umma_commit(bar(B_Q_EMPTY0 + qb));
                }
                if (!ok) break;
                for (int pp = 0; pp < npipe; ++pp) umma_commit(bar(B_O_FULL + pp));
            }
            // every MMA issued so far has retired before the tensor memory is freed
            umma_commit(bar(B_MMA_DONE));
            mbar_wait(bar(B_MMA_DONE), 0, abort_flag, nullptr, 0);
        }
    } else if (warp >= 8) {
        // ============ epilogue: output, group sum, top-k (128 thr) ============
        setmaxnreg_dec<kRegsEpilogue>();
        const int ew = warp - 8;                   // TMEM lane quadrant
        const int erow = ew * 32 + lane;
        const uint32_t lane_off = (uint32_t)(ew * 32) << 16;
        const int cap = p.score_cap;
        float* score = p.score_in_smem ? reinterpret_cast<float*>(smem + p.off_score) + ew * cap
                                       : p.score_gmem + ((size_t)blockIdx.x * 4 + ew) * cap;
        float* mbw = reinterpret_cast<float*>(smem + p.off_rowstat) + 2 * 2 * 2 * 128 + ew * 128;
        const uint64_t out_policy = l2_policy_evict_first();   // attention_out is written once
        int tcount = 0;
        const int eh = erow % G;
        const int etok = erow / G;

        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
            const AttnTile t = p.tiles[tile];
            const int slot = tcount & 1;
            for (int pp = 0; pp < npipe; ++pp) {
                mbar_wait(bar(B_ROW_DONE + 2 * pp + slot), (tcount >> 1) & 1, abort_flag, p.err,
                          kErrTimeoutBase + 14);
                mbar_wait(bar(B_O_FULL + pp), tcount & 1, abort_flag, p.err, kErrTimeoutBase + 12);
                tc_fence_after();
                // O (tensor memory) / L -> attention_out
                const int tok = pp * TT + etok;
                const bool valid = (erow < TT * G) && (tok < t.ntok) &&
                                   nsa_index_ok(t.q_row0 + tok < p.rows_q, p.err, 1);
                const int nvis = valid ? nvis_of(t.t0 + tok, p.l, p.d, t.n_cmp) : 0;
                const float Lr = rowstat[((pp * 2 + slot) * 2 + 1) * 128 + erow];
                // rows that attend to nothing write zeros (their O may never have been
                // written: select, do not multiply)
                const bool live = nvis > 0 && Lr > 0.f;
                const float inv = live ? 1.f / Lr : 0.f;
                T* orow = reinterpret_cast<T*>(p.out) +
                          ((size_t)(t.q_row0 + tok) * p.n1 + (size_t)t.group * G + eh) * p.d2;
                const uint32_t obase = tmem + lane_off + (pp ? p.tm_o[1] : p.tm_o[0]);
                for (int c = 0; c < p.d2 / 16; ++c) {
                    uint32_t r[16];
                    tmem_ld16(obase + c * 16, r);
                    tmem_wait_ld_regs<16>(r);
                    if (valid) {
                        uint4 w0, w1;
                        float f[16];
#pragma unroll
                        for (int q = 0; q < 16; ++q) f[q] = live ? __uint_as_float(r[q]) * inv : 0.f;
                        w0.x = pack2<T>(f[0], f[1]);
                        w0.y = pack2<T>(f[2], f[3]);
                        w0.z = pack2<T>(f[4], f[5]);
                        w0.w = pack2<T>(f[6], f[7]);
                        w1.x = pack2<T>(f[8], f[9]);
                        w1.y = pack2<T>(f[10], f[11]);
                        w1.z = pack2<T>(f[12], f[13]);
                        w1.w = pack2<T>(f[14], f[15]);
                        st_global_v4_hint(orow + c * 16, w0, out_policy);
                        st_global_v4_hint(orow + c * 16 + 8, w1, out_policy);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_O_EMPTY + pp));
            }

            // steps 4-5 from the scratch rows, then step 7; one warp per token
            for (int tau = ew; tau < t.ntok; tau += 4) {
                const int pp = tau / TT;
                const int tl = tau - pp * TT;
                const int tp = t.t0 + tau;
                if (!nsa_index_ok(t.q_row0 + tau < p.rows_q && t.group < p.n2, p.err, 2)) continue;
                int32_t* dst = p.topk + ((size_t)(t.q_row0 + tau) * p.n2 + t.group) * p.count;
                const int nv = nvis_of(tp, p.l, p.d, t.n_cmp);
                bool empty = nv == 0;
                const uint32_t* trow = nullptr;
                if constexpr (kMask) {
                    // a token whose visible blocks are all masked attends to nothing; its
                    // heads share the mask row, so its first head's softmax sum is 0
                    if (!empty && p.am_bits != nullptr)
                        empty = rowstat[((pp * 2 + slot) * 2 + 1) * 128 + tl * G] == 0.f;
                    if (p.tm_bits != nullptr) trow = p.tm_bits + (size_t)(t.tloc0 + tau) * p.tm_words;
                }
                if (empty) {
                    for (int j = lane; j < p.count; j += 32) dst[j] = -1;
                    continue;
                }
                const int ncand = min(t.n_sel, tp / p.lp + 1);
                // anchors past nkv*NJ + NJC collect no tap from a visible block
                const int jn = min(ncand, t.nkv * NJ + NJC);
                const float* base = p.band + (((size_t)blockIdx.x * npipe + pp) * 2 + slot) * (size_t)p.region;
                if constexpr (kTwoPass) {
                    // the token's scores were summed over its heads by the softmax warps:
                    // [chunk][token][NJC] in the slot; lane l takes anchors 4l..4l+3 of every 128
                    for (int j0 = 0; j0 < jn; j0 += 128) {
                        const int j4 = j0 + 4 * lane;
                        if (j4 < jn) {
                            const int c = j4 / NJC;
                            const float4 v4 = __ldcg(reinterpret_cast<const float4*>(
                                base + ((size_t)c * TT + tl) * NJC + (j4 - c * NJC)));
                            *reinterpret_cast<float4*>(score + j4) = v4;
                        }
                    }
                } else {
                    const float* rs = rowstat + (pp * 2 + slot) * 2 * 128 + tl * G;
                    // the token's heads' normalisers m_ref + log2 L, once
                    for (int hh = lane; hh < G; hh += 32) {
                        const float Lh = rs[128 + hh];
                        mbw[hh] = (Lh > 0.f) ? rs[hh] + lg2(Lh) : INFINITY;
                    }
                    __syncwarp();
                    // P_slc'[j] = sum_h 2^(m_c - m_ref - log2 L) x banded value, where m_c
                    // is the reference the value's chunk was written against (steps 4-5).
                    // Lane l takes anchors 4l..4l+3 of every 128 (in one chunk, NJC % 4 == 0)
                    // and loops over the heads, eight at a time for loads in flight.
                    const float* wbase = base + p.capj + (size_t)(tl * G) * p.capc;
                    // (measured on B200: the chunk weights computed here, with their
                    // references loaded next to the banded values, beat a per-step weight
                    // table filled first, which serialises two L2 round trips per step)
                    for (int j0 = 0; j0 < jn; j0 += 128) {
                        const int j4 = j0 + 4 * lane;
                        const bool live = j4 < jn;
                        const int c = j4 / NJC;                     // chunk of the four anchors
                        const float* bp = base + ((size_t)c * 128 + tl * G) * NJC + (j4 - c * NJC);
                        const float* wp = wbase + c;
                        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                        int hh = 0;
                        for (; hh + 8 <= G; hh += 8) {
                            float4 bv[8];
                            float mv[8];
    #pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                bv[u] = live ? __ldcg(reinterpret_cast<const float4*>(bp + (size_t)(hh + u) * NJC))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
                                mv[u] = live ? __ldcg(wp + (size_t)(hh + u) * p.capc) : 0.f;
                            }
    #pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const float w = live ? ex2(mv[u] - mbw[hh + u]) : 0.f;
                                acc.x = fmaf(w, bv[u].x, acc.x);
                                acc.y = fmaf(w, bv[u].y, acc.y);
                                acc.z = fmaf(w, bv[u].z, acc.z);
                                acc.w = fmaf(w, bv[u].w, acc.w);
                            }
                        }
                        for (; hh < G; ++hh) {
                            if (live) {
                                const float4 b1 = __ldcg(reinterpret_cast<const float4*>(bp + (size_t)hh * NJC));
                                const float w = ex2(__ldcg(wp + (size_t)hh * p.capc) - mbw[hh]);
                                acc.x = fmaf(w, b1.x, acc.x);
                                acc.y = fmaf(w, b1.y, acc.y);
                                acc.z = fmaf(w, b1.z, acc.z);
                                acc.w = fmaf(w, b1.w, acc.w);
                            }
                        }
                        if (live) *reinterpret_cast<float4*>(score + j4) = acc;
                    }
                }
                __syncwarp();
                warp_topk<kMask>(score, ncand, jn, p.count, dst, lane, trow);
                __syncwarp();   // the score row is free for the next token
            }
            // every token of the item is done: the slot's scratch is dead, so its
            // lines leave L2 without a write-back; then slot and row statistics
            // are free
            named_bar_sync(2, 128);
            if (t.nkv > 0) {
                // (two passes: one row of scores per token, no chunk references)
                const size_t band_bytes = (size_t)(t.nkv * NCH + 1) * (kTwoPass ? TT : 128) * NJC * 4;
                for (int pp = 0; pp < npipe; ++pp) {
                    const char* sb0 = reinterpret_cast<const char*>(
                        p.band + (((size_t)blockIdx.x * npipe + pp) * 2 + slot) * (size_t)p.region);
                    for (size_t o = (size_t)(warp - 8) * 32 + lane; o * 128 < band_bytes; o += 128)
                        discard_l2_line(sb0 + o * 128);
                    const size_t mref_bytes = kTwoPass ? 0 : (size_t)128 * p.capc * 4;
                    const char* mb0 = sb0 + (size_t)p.capj * 4;
                    for (size_t o = (size_t)(warp - 8) * 32 + lane; o * 128 < mref_bytes; o += 128)
                        discard_l2_line(mb0 + o * 128);
                }
            }
            __syncwarp();
            if (lane == 0)
                for (int pp = 0; pp < npipe; ++pp) mbar_arrive(bar(B_SCR_EMPTY + 2 * pp + slot));
        }
    } else {
        // ========== softmax, P, banded values (128 threads per pipeline) ==========
        setmaxnreg_inc<kRegsSoftmax>();
        const int pp = warp >> 2;                  // pipeline
        if (pp < npipe) {
            const int wq = warp & 3;               // TMEM lane quadrant
            const int row = wq * 32 + lane;        // tile row = TMEM lane
            const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
            const int a = p.a, bb = p.b;
            const float c2 = p.scale_log2;
            float wband[NTAP];
#pragma unroll
            for (int u = 0; u < NTAP; ++u) {
                // multiplicity of m + n = u with m < a, n < b (the double sum of step 4)
                const int c = min(min(u, a - 1), min(bb - 1, a + bb - 2 - u)) + 1;
                wband[u] = (u <= a + bb - 2) ? (float)c : 0.f;
            }
            const int h = row % G;
            const int tok_t = row / G;
            // scores in "exponent units": x = s * ce - m_ref.  With a positive
            // scale the raw scores are used as they are (ce = c2); a zero or
            // negative scale first multiplies them in (ce = 1).
            const bool pos_scale = c2 > 0.f;
            const float ce = pos_scale ? c2 : 1.f;
            const float2 ce2 = make_float2(ce, ce);
            int scnt = 0, pcnt = 0, tcount = 0;
            const uint32_t tm_sp = tmem + lane_off + (pp ? p.tm_s[1] : p.tm_s[0]);
            const uint32_t tm_op = tmem + lane_off + (pp ? p.tm_o[1] : p.tm_o[0]);

            for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
                const AttnTile t = p.tiles[tile];
                const int tok = pp * TT + tok_t;
                const bool valid = (row < TT * G) && (tok < t.ntok);
                const int tpos = t.t0 + tok;
                const int nvis = valid ? nvis_of(tpos, p.l, p.d, t.n_cmp) : 0;
                const int slot = tcount & 1;
                const uint32_t* arow = nullptr;
                if constexpr (kMask)
                    arow = (valid && p.am_bits != nullptr) ? p.am_bits + (size_t)(t.tloc0 + tok) * p.am_words
                                                           : nullptr;
                // this slot's scratch: banded values [chunk][row][NJC], then the chunk
                // references [row][chunk]
                float* sbase_g = p.band + (((size_t)blockIdx.x * npipe + pp) * 2 + slot) * (size_t)p.region;
                float* wrow = sbase_g + p.capj + (size_t)row * p.capc;
                // the epilogue has finished with this slot (item tcount - 2)
                mbar_wait(bar(B_SCR_EMPTY + 2 * pp + slot), ((tcount >> 1) & 1) ^ 1, abort_flag, p.err,
                          kErrTimeoutBase + 13);

                if constexpr (kTwoPass) {
                    // a score chunk in exponent units (x = s * ce), masked columns -inf
                    auto load_chunk = [&](uint32_t sbase, int i, int c, int lim, float (&sx)[CH]) {
                        uint32_t rb[CH];
                        tmem_ld_n<CH>(sbase + c * CH, rb);
                        tmem_wait_ld_regs<CH>(rb);
#pragma unroll
                        for (int e = 0; e < CH; ++e) sx[e] = __uint_as_float(rb[e]) * (pos_scale ? 1.f : c2);
                        const int cl = lim - c * CH;
                        if (cl < CH) {
#pragma unroll
                            for (int e = 0; e < CH; ++e) sx[e] = (e < cl) ? sx[e] : -INFINITY;
                        }
                        if constexpr (kMask) {
                            if (arow != nullptr) {
                                const int col0 = i * NKV + c * CH;
                                const int w0 = col0 >> 5, b0 = col0 & 31;
                                const uint32_t a0 = arow[w0], a1 = arow[w0 + 1], a2 = arow[w0 + 2];
                                const uint32_t lo = __funnelshift_r(a0, a1, b0), hi = __funnelshift_r(a1, a2, b0);
#pragma unroll
                                for (int e = 0; e < CH; ++e)
                                    if (((e < 32 ? lo >> e : hi >> (e - 32)) & 1u) != 0u) sx[e] = -INFINITY;
                            }
                        }
                    };
                    // ---- pass 1: the row's exact maximum m and sum L = sum 2^(x - m) ----
                    float m = -INFINITY, L = 0.f;
                    for (int i = 0; i < t.nkv; ++i) {
                        const int sb = scnt % nsb;
                        mbar_wait(bar(B_S_FULL + 2 * pp + sb), (scnt / nsb) & 1, abort_flag, p.err,
                                  kErrTimeoutBase + 10);
                        tc_fence_after();
                        const uint32_t sbase = tm_sp + sb * 128;
                        const int lim = nvis - i * NKV;
#pragma unroll 1
                        for (int c = 0; c < NCH; ++c) {
                            float sx[CH];
                            load_chunk(sbase, i, c, lim, sx);
                            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                            for (int e = 0; e + 8 <= CH; e += 8) {
                                mx4[0] = fmax3(mx4[0], sx[e + 0], sx[e + 1]);
                                mx4[1] = fmax3(mx4[1], sx[e + 2], sx[e + 3]);
                                mx4[2] = fmax3(mx4[2], sx[e + 4], sx[e + 5]);
                                mx4[3] = fmax3(mx4[3], sx[e + 6], sx[e + 7]);
                            }
                            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * ce;
                            if (mx > m) {
                                L = (m == -INFINITY) ? 0.f : L * ex2(m - mx);
                                m = mx;
                            }
                            if (m > -INFINITY) {
                                const float2 nm2 = make_float2(-m, -m);
                                float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                                  make_float2(0.f, 0.f)};
#pragma unroll
                                for (int e = 0; e < CH; e += 2) {
                                    const float2 x = ffma2(make_float2(sx[e], sx[e + 1]), ce2, nm2);
                                    acc2[(e >> 1) & 3] = fadd2(acc2[(e >> 1) & 3], make_float2(ex2(x.x), ex2(x.y)));
                                }
                                const float2 t01 = fadd2(acc2[0], acc2[1]), t23 = fadd2(acc2[2], acc2[3]);
                                L += (t01.x + t01.y) + (t23.x + t23.y);
                            }
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B_P_FULL + pp));   // the score buffer is read
                        ++scnt;
                        ++pcnt;
                    }
                    // P~ = 2^(x - m) relative to the exact maximum (the maximum itself is 1,
                    // exact in the storage dtype) feeds P V; the band values take P~ / L in
                    // fp32, the normalised P of step 2.  0 for a row that attends to nothing.
                    const float mref = (L > 0.f) ? m : INFINITY;
                    const float inv_l = (L > 0.f) ? 1.f / L : 0.f;
                    const float2 nmb2 = make_float2(-mref, -mref);
                    // ---- pass 2: P, P V, and the band values summed over the token's G heads ----
                    // The heads of a token are G adjacent lanes (G a power of two <= 32): a
                    // transposing butterfly leaves lane h with anchors [h NJC/G, (h+1) NJC/G)
                    // of the token's sum, written to the slot as [chunk][token][NJC].
                    auto reduce_store = [&](float (&v)[NJC], int q) {
                        int off = 0;
#pragma unroll
                        for (int st = 0, half = NJC / 2; half >= 1; ++st, half >>= 1) {
                            const int dist = G >> (st + 1);
                            if (dist == 0) break;
                            const bool upper = (lane & dist) != 0;
#pragma unroll
                            for (int e = 0; e < half; ++e) {
                                const float send = upper ? v[e] : v[e + half];
                                const float keep = upper ? v[e + half] : v[e];
                                v[e] = keep + __shfl_xor_sync(0xffffffffu, send, dist);
                            }
                            if (upper) off += half;
                        }
                        // G > NJC: the lanes that share a set of anchors finish the sum
                        for (int dist = G / (2 * NJC); dist >= 1; dist >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], dist);
                        const int per = NJC >= G ? NJC / G : 1;
                        const bool writer = NJC >= G || (h % (G / NJC)) == 0;
                        const bool in_slot = nsa_index_ok((size_t)(q + 1) * TT * NJC <= (size_t)p.capj, p.err, 4);
                        if (valid && writer && in_slot) {
                            float* dst = sbase_g + ((size_t)q * TT + tok_t) * NJC + off;
#pragma unroll
                            for (int e = 0; e < NJC; ++e)
                                if (e < per) __stcg(dst + e, v[e]);
                        }
                    };
                    float carry[NCARRY];
#pragma unroll
                    for (int k = 0; k < NCARRY; ++k) carry[k] = 0.f;
                    for (int i = 0; i < t.nkv; ++i) {
                        const int sb = scnt % nsb;
                        mbar_wait(bar(B_S_FULL + 2 * pp + sb), (scnt / nsb) & 1, abort_flag, p.err,
                                  kErrTimeoutBase + 10);
                        tc_fence_after();
                        const uint32_t sbase = tm_sp + sb * 128;
                        const int lim = nvis - i * NKV;
#pragma unroll 1
                        for (int c = 0; c < NCH; ++c) {
                            float sx[CH];
                            load_chunk(sbase, i, c, lim, sx);
#pragma unroll
                            for (int e = 0; e < CH; e += 2) {
                                const float2 x = ffma2(make_float2(sx[e], sx[e + 1]), ce2, nmb2);
                                sx[e] = ex2(x.x);
                                sx[e + 1] = ex2(x.y);
                            }
                            {
                                uint32_t pk[CH / 2];
#pragma unroll
                                for (int e = 0; e < CH / 2; ++e) pk[e] = pack2<T>(sx[2 * e], sx[2 * e + 1]);
                                tmem_st_n<CH / 2>(sbase + c * (CH / 2), pk);
                            }
                            float v[NJC];
#pragma unroll
                            for (int jj = 0; jj < NJC; ++jj) {
                                float acc = 0.f;
#pragma unroll
                                for (int u = 0; u < NTAP; ++u) {
                                    const int x = A * jj - u;
                                    const float pv = (x >= 0) ? sx[x >= 0 ? x : 0] : carry[x < 0 ? (-x - 1) : 0];
                                    acc = fmaf(wband[u], pv, acc);
                                }
                                v[jj] = acc;
                            }
#pragma unroll
                            for (int k = 0; k < NCARRY; ++k) carry[k] = sx[CH - 1 - k];
#pragma unroll
                            for (int jj = 0; jj < NJC; ++jj) v[jj] *= inv_l;
                            reduce_store(v, i * NCH + c);
                        }
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B_P_FULL + pp));
                        ++scnt;
                        ++pcnt;
                    }
                    if (t.nkv > 0) {
                        // the first anchors past the last tile still collect taps from it
                        float v[NJC];
#pragma unroll
                        for (int jj = 0; jj < NJC; ++jj) {
                            float acc = 0.f;
#pragma unroll
                            for (int u = 0; u < NTAP; ++u) {
                                const int x = A * jj - u;
                                if (x < 0) acc = fmaf(wband[u], carry[-x - 1 >= 0 ? -x - 1 : 0], acc);
                            }
                            v[jj] = acc * inv_l;
                        }
                        reduce_store(v, t.nkv * NCH);
                    }
                    if (valid && nsa_index_ok(t.q_row0 + tok < p.rows_q, p.err, 3)) {
                        const size_t si = ((size_t)(t.q_row0 + tok) * p.n1 + (size_t)t.group * G + h) * 8;
                        const float mo = (m == -INFINITY) ? -INFINITY : m * 0.69314718055994530942f;
                        const float4 mv = make_float4(mo, mo, mo, mo);
                        const float4 lv = make_float4(L, L, L, L);
                        reinterpret_cast<float4*>(p.smax + si)[0] = mv;
                        reinterpret_cast<float4*>(p.smax + si)[1] = mv;
                        reinterpret_cast<float4*>(p.ssum + si)[0] = lv;
                        reinterpret_cast<float4*>(p.ssum + si)[1] = lv;
                    }
                    // the epilogue divides O by L (0 for a row that attends to nothing)
                    rowstat[((pp * 2 + slot) * 2 + 0) * 128 + row] = m;
                    rowstat[((pp * 2 + slot) * 2 + 1) * 128 + row] = L;
                    __threadfence_block();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(B_ROW_DONE + 2 * pp + slot));
                    continue;
                }

                float m_ref = -INFINITY, m_true = -INFINITY, L = 0.f;
                float carry[NCARRY];   // carry[k] = P of the column 1 + k before the chunk
#pragma unroll
                for (int k = 0; k < NCARRY; ++k) carry[k] = 0.f;

                for (int i = 0; i < t.nkv; ++i) {
                    const int sb = scnt % nsb;
                    mbar_wait(bar(B_S_FULL + 2 * pp + sb), (scnt / nsb) & 1, abort_flag, p.err,
                              kErrTimeoutBase + 10);
                    tc_fence_after();
                    const uint32_t sbase = tm_sp + sb * 128;
                    const int lim = nvis - i * NKV;   // visible columns of this tile
                    uint32_t rb[CH];
                    if constexpr (kPrefetch) tmem_ld_n<CH>(sbase, rb);
                    // a rolled loop: measured on B200, unrolling the chunks grows the
                    // hot code past what the instruction caches hold with the other
                    // roles running on the same SM (128K workload 46.7 -> 41.9 ms rolled)
#pragma unroll 1
                    for (int c = 0; c < NCH; ++c) {
                        float s[CH];
                        if constexpr (!kPrefetch) tmem_ld_n<CH>(sbase + c * CH, rb);
                        tmem_wait_ld_regs<CH>(rb);
#pragma unroll
                        for (int e = 0; e < CH; ++e) s[e] = __uint_as_float(rb[e]);
                        const int cl = lim - c * CH;   // visible columns of this chunk
                        if (!pos_scale) {
#pragma unroll
                            for (int e = 0; e < CH; ++e) s[e] *= c2;
                        }
                        if (cl < CH) {
#pragma unroll
                            for (int e = 0; e < CH; ++e) s[e] = (e < cl) ? s[e] : -INFINITY;
                        }
                        if constexpr (kMask) {
                            // atten_mask (step 1), bit-packed: a set bit removes a visible
                            // block; the chunk's CH <= 64 bits from a three-word window
                            if (arow != nullptr) {
                                const int col0 = i * NKV + c * CH;
                                const int w0 = col0 >> 5, b0 = col0 & 31;
                                const uint32_t a0 = arow[w0], a1 = arow[w0 + 1], a2 = arow[w0 + 2];
                                const uint32_t lo = __funnelshift_r(a0, a1, b0), hi = __funnelshift_r(a1, a2, b0);
#pragma unroll
                                for (int e = 0; e < CH; ++e)
                                    if (((e < 32 ? lo >> e : hi >> (e - 32)) & 1u) != 0u) s[e] = -INFINITY;
                            }
                        }
                        // chunk maximum: independent chains of 3-input max
                        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                        for (int e = 0; e + 8 <= CH; e += 8) {
                            mx4[0] = fmax3(mx4[0], s[e + 0], s[e + 1]);
                            mx4[1] = fmax3(mx4[1], s[e + 2], s[e + 3]);
                            mx4[2] = fmax3(mx4[2], s[e + 4], s[e + 5]);
                            mx4[3] = fmax3(mx4[3], s[e + 6], s[e + 7]);
                        }
                        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * ce;
                        m_true = fmaxf(m_true, mx);
                        const bool need = (m_ref == -INFINITY) ? (mx > -INFINITY) : (mx > m_ref + kRescaleLog2);
                        if (__any_sync(0xffffffffu, need)) {
                            // move the reference maximum: everything summed or written
                            // relative to the old one is scaled by 2^(old - new)
                            const float m_new = need ? mx : m_ref;
                            const float f = need ? ((m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new)) : 1.f;
                            L *= f;
#pragma unroll
                            for (int k = 0; k < NCARRY; ++k) carry[k] *= f;
                            if (c > 0) {
                                tmem_wait_st();
#pragma unroll
                                for (int c0 = 0; c0 < NCH; ++c0)
                                    if (c0 < c) tmem_scale_packed<T, CH / 2>(sbase + c0 * (CH / 2), f);
                            }
                            if (i > 0) {
                                // P V of the previous tile has completed before O is touched
                                mbar_wait(bar(B_P_EMPTY + pp), (pcnt - 1) & 1, abort_flag, p.err,
                                          kErrTimeoutBase + 11);
                                tc_fence_after();
                                tmem_scale_f32(tm_op, p.d2, f);
                            }
                            m_ref = m_new;
                        }
                        // the next chunk's load runs while this one's P and band values
                        // are computed (issued after the scaling above, which waits for
                        // its own tensor-memory loads)
                        if constexpr (kPrefetch) {
                            if (c + 1 < NCH) tmem_ld_n<CH>(sbase + (c + 1) * CH, rb);
                        }
                        const float mr = (m_ref == -INFINITY) ? 0.f : m_ref;
                        const float2 nm2 = make_float2(-mr, -mr);
                        // P = 2^(x - m_ref) in fp32; partial sums in pairs
                        float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                          make_float2(0.f, 0.f)};
#pragma unroll
                        for (int e = 0; e < CH; e += 2) {
                            const float2 x = ffma2(make_float2(s[e], s[e + 1]), ce2, nm2);
                            s[e] = ex2(x.x);
                            s[e + 1] = ex2(x.y);
                            acc2[(e >> 1) & 3] = fadd2(acc2[(e >> 1) & 3], make_float2(s[e], s[e + 1]));
                        }
                        const float2 t01 = fadd2(acc2[0], acc2[1]), t23 = fadd2(acc2[2], acc2[3]);
                        L += (t01.x + t01.y) + (t23.x + t23.y);
                        // P in the storage dtype over the score columns it came from
                        {
                            uint32_t pk[CH / 2];
#pragma unroll
                            for (int e = 0; e < CH / 2; ++e) pk[e] = pack2<T>(s[2 * e], s[2 * e + 1]);
                            tmem_st_n<CH / 2>(sbase + c * (CH / 2), pk);
                        }
                        // step 4 on the fp32 P: anchors A*jj of this chunk; taps reach
                        // back into the previous chunk through `carry`
                        float v[NJC];
#pragma unroll
                        for (int jj = 0; jj < NJC; ++jj) {
                            float acc = 0.f;
#pragma unroll
                            for (int u = 0; u < NTAP; ++u) {
                                const int x = A * jj - u;
                                const float pv = (x >= 0) ? s[x >= 0 ? x : 0] : carry[x < 0 ? (-x - 1) : 0];
                                acc = fmaf(wband[u], pv, acc);
                            }
                            v[jj] = acc;
                        }
#pragma unroll
                        for (int k = 0; k < NCARRY; ++k) carry[k] = s[CH - 1 - k];
                        // (debug builds: the chunk stays inside the slot's scratch)
                        const bool in_slot =
                            nsa_index_ok((i * NCH + c + 1) * 128 * NJC <= p.capj && i * NCH + c < p.capc, p.err, 4);
                        if (valid && in_slot) __stcg(wrow + i * NCH + c, mr);
                        if (valid && in_slot) {
                            // a warp writes its 32 rows' values of the chunk contiguously
                            float4* bd = reinterpret_cast<float4*>(
                                sbase_g + ((size_t)(i * NCH + c) * 128 + row) * NJC);
#pragma unroll
                            for (int q4 = 0; q4 < NJC / 4; ++q4)
                                __stcg(bd + q4, make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]));
                        }
                    }

                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(B_P_FULL + pp));
                    ++scnt;
                    ++pcnt;
                }
                const float mr = (m_ref == -INFINITY) ? 0.f : m_ref;
                if (t.nkv > 0 && valid) {
                    // the first anchors past the last tile still collect taps from it
                    float v[NJC];
#pragma unroll
                    for (int jj = 0; jj < NJC; ++jj) {
                        float acc = 0.f;
#pragma unroll
                        for (int u = 0; u < NTAP; ++u) {
                            const int x = A * jj - u;
                            if (x < 0) acc = fmaf(wband[u], carry[-x - 1 >= 0 ? -x - 1 : 0], acc);
                        }
                        v[jj] = acc;
                    }
                    float4* bd = reinterpret_cast<float4*>(sbase_g + ((size_t)t.nkv * NCH * 128 + row) * NJC);
#pragma unroll
                    for (int q4 = 0; q4 < NJC / 4; ++q4)
                        __stcg(bd + q4, make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]));
                    __stcg(wrow + t.nkv * NCH, mr);
                }
                if (valid && nsa_index_ok(t.q_row0 + tok < p.rows_q, p.err, 3)) {
                    // softmax_max / softmax_sum: exact maximum (natural units) and the
                    // sum of exp(s - max)
                    const size_t si = ((size_t)(t.q_row0 + tok) * p.n1 + (size_t)t.group * G + h) * 8;
                    const float mo = (m_true == -INFINITY) ? -INFINITY : m_true * 0.69314718055994530942f;
                    const float lt = (L > 0.f) ? L * ex2(mr - m_true) : 0.f;
                    const float4 mv = make_float4(mo, mo, mo, mo);
                    const float4 lv = make_float4(lt, lt, lt, lt);
                    reinterpret_cast<float4*>(p.smax + si)[0] = mv;
                    reinterpret_cast<float4*>(p.smax + si)[1] = mv;
                    reinterpret_cast<float4*>(p.ssum + si)[0] = lv;
                    reinterpret_cast<float4*>(p.ssum + si)[1] = lv;
                }
                rowstat[((pp * 2 + slot) * 2 + 0) * 128 + row] = mr;
                rowstat[((pp * 2 + slot) * 2 + 1) * 128 + row] = L;
                __threadfence_block();   // scratch rows and statistics before the hand-off
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_ROW_DONE + 2 * pp + slot));
            }
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
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// A byte mask (rows x s2, nonzero = set) to bit rows of `words` 32-bit words:
// bit j of row r = src[r][j] for j < ncols, 0 beyond.  One warp per (row,
// 32 words): lane k reads byte 32 w + k of each word w in turn (coalesced),
// a ballot forms the word, and lane w % 32 stores it.
__global__ void pack_mask_kernel(const uint8_t* __restrict__ src, long long s2, int ncols, int rows, int words,
                                 uint32_t* __restrict__ dst) {
    const int lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int wbase = blockIdx.y * 32;
    const uint8_t* row = src + r * s2;
    uint32_t mine = 0;
    for (int k = 0; k < 32; ++k) {
        const int col = (wbase + k) * 32 + lane;
        const bool set = col < ncols && row[col] != 0;
        const uint32_t word = __ballot_sync(0xffffffffu, set);
        if (lane == k) mine = word;
    }
    if (wbase + lane < words) dst[r * words + wbase + lane] = mine;
}

cudaError_t launch_pack_mask(const uint8_t* src, long long s2, int ncols, int rows, int words, uint32_t* dst,
                             cudaStream_t st) {
    if (rows <= 0 || words <= 0) return cudaSuccess;
    dim3 grid((rows + 7) / 8, (words + 31) / 32);
    pack_mask_kernel<<<grid, 256, 0, st>>>(src, s2, ncols, rows, words, dst);
    return cudaGetLastError();
}

template <typename T, int A, bool kMask, bool kTwoPass>
static cudaError_t launch_t(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, int grid, cudaStream_t st) {
    auto kern = nsa_cmp_attn_kernel<T, A, kMask, kTwoPass>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kAttnThreads, p.smem_bytes, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

template <typename T, bool kMask>
static cudaError_t launch_a(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, int grid, cudaStream_t st) {
    // two passes (head sums on chip) for 128-block KV tiles and G a power of two <= 32
    if (p.two_pass) {
        switch (p.a) {
            case 1: return launch_t<T, 1, kMask, true>(p, tq, tk, tv, grid, st);
            case 2: return launch_t<T, 2, kMask, true>(p, tq, tk, tv, grid, st);
            case 4: return launch_t<T, 4, kMask, true>(p, tq, tk, tv, grid, st);
            case 8: return launch_t<T, 8, kMask, true>(p, tq, tk, tv, grid, st);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (p.a) {
        case 1: return launch_t<T, 1, kMask, false>(p, tq, tk, tv, grid, st);
        case 2: return launch_t<T, 2, kMask, false>(p, tq, tk, tv, grid, st);
        case 3: return launch_t<T, 3, kMask, false>(p, tq, tk, tv, grid, st);
        case 4: return launch_t<T, 4, kMask, false>(p, tq, tk, tv, grid, st);
        case 5: return launch_t<T, 5, kMask, false>(p, tq, tk, tv, grid, st);
        case 6: return launch_t<T, 6, kMask, false>(p, tq, tk, tv, grid, st);
        case 7: return launch_t<T, 7, kMask, false>(p, tq, tk, tv, grid, st);
        case 8: return launch_t<T, 8, kMask, false>(p, tq, tk, tv, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_attention(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, int grid, cudaStream_t st) {
    // the masked kernel only where a mask is given: the unmasked one is unchanged
    if (p.am_bits != nullptr || p.tm_bits != nullptr)
        return p.dtype == 0 ? launch_a<__nv_bfloat16, true>(p, tq, tk, tv, grid, st)
                            : launch_a<__half, true>(p, tq, tk, tv, grid, st);
    return p.dtype == 0 ? launch_a<__nv_bfloat16, false>(p, tq, tk, tv, grid, st)
                        : launch_a<__half, false>(p, tq, tk, tv, grid, st);
}

}  // namespace nsa
