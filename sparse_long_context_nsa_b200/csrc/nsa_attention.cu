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
// step 5 is a sum over neighbouring rows.  Two passes over the compressed
// keys per tile, because step 5 adds *normalised* probabilities of different
// heads and a head's normaliser is only known at the end of its row:
//   pass A  S = Q K^T (tcgen05.mma, operands in shared memory, fp32 in tensor
//           memory); online max / sum in registers -> exact m and L per row;
//           softmax_max / softmax_sum are written here.
//   pass B  S = Q K^T again; P = 2^(s*scale*log2e - m - log2 L) in fp32
//           registers; P (storage dtype) -> tensor memory -> O += P V with the
//           A operand read from tensor memory; from the fp32 P the banded sum
//           of step 4 goes to a shared-memory staging ring.
// A 128-column score tile (a >= 4) is read from tensor memory in two halves:
// the second half's load is in flight while the first half's exponentials
// run.
// Epilogue warps, concurrently with the next tile's passes: sum the staged
// band values over the G rows of each token into a per-token score buffer
// (step 5), read O out of tensor memory, and pick the top-k (step 7).
// Warp roles (384 threads, three warpgroups): warps 0-3 softmax (warp w owns
// TMEM lanes 32w..32w+31 = tile rows), warps 4-7 epilogue (same lane
// quadrants), warp 8 TMA producer, warp 9 MMA issuer (and tensor-memory
// owner), warps 10-11 idle.  Registers move from the third and second
// warpgroups to the softmax warpgroup with setmaxnreg.  One persistent CTA
// per SM.
// Q (double-buffered), K and V are staged by TMA with 128-byte swizzle; K and
// V share one ring of slots.  Every mbarrier wait is bounded; a timeout sets
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

int attention_kv_cols(int a) { return kv_cols_for(a); }

enum BarId {
    B_Q_FULL0 = 0,
    B_Q_FULL1,
    B_Q_EMPTY0,
    B_Q_EMPTY1,
    B_S_FULL0,
    B_S_FULL1,
    B_S_EMPTY0,
    B_S_EMPTY1,
    B_P_FULL,
    B_P_EMPTY,
    B_O_FULL,
    B_O_EMPTY,
    B_STG_FULL0,
    B_STG_FULL1,
    B_STG_EMPTY0,
    B_STG_EMPTY1,
    B_MMA_DONE,
    B_SLOT_FULL0,                     // + slot
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

// k-th largest key (fp32 bit pattern) of sc[0 .. ncand) held in registers,
// NR keys per lane (key i of a lane belongs to j = lane + 32 i); keys at
// j >= lim are 0.  Bitwise search from the top bit down.
template <int NR, bool kMask>
__device__ __forceinline__ uint32_t kth_key_regs(const float* sc, int ncand, int lim, int k, int lane,
                                                 const uint8_t* trow) {
    uint32_t key[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
        const int j = lane + 32 * i;
        bool in = j < lim;
        if constexpr (kMask) in = in && !(trow && trow[j]);
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
    }
    return thr;
}

// Top-k of one token's group scores (step 7), one warp.  Candidates are
// j < ncand; scores for j >= jcov are 0 (no visible block reaches them).
// Exact k-th largest key by a bitwise search over the fp32 bit patterns
// (scores are >= 0, so the bit patterns order like the values), then an
// ordered ballot scan keeps every key above it plus the earliest ties, which
// also lists the indices in ascending order.  With a topk_mask row (kMask),
// candidates whose mask byte is set are out of the set (step 6).
template <bool kMask>
__device__ __forceinline__ void warp_topk(const float* sc, int ncand, int jcov, int count,
                                          int32_t* dst, int lane, const uint8_t* trow) {
    auto masked = [&](int j) {
        if constexpr (kMask) return trow != nullptr && trow[j] != 0;
        return false;
    };
    int n_in = ncand;
    if constexpr (kMask) {
        if (trow) {
            int nm = 0;
            for (int j = lane; j < ncand; j += 32) nm += trow[j] ? 1 : 0;
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

// Online max / sum update (log2 domain) with score columns [C0, C0 + W).
template <int C0, int W, int N>
__device__ __forceinline__ void online_update(const float (&s)[N], float ce, float& m, float& L) {
    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < W; c += 8) {
        mx4[0] = fmax3(mx4[0], s[C0 + c + 0], s[C0 + c + 1]);
        mx4[1] = fmax3(mx4[1], s[C0 + c + 2], s[C0 + c + 3]);
        mx4[2] = fmax3(mx4[2], s[C0 + c + 4], s[C0 + c + 5]);
        mx4[3] = fmax3(mx4[3], s[C0 + c + 6], s[C0 + c + 7]);
    }
    const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * ce;
    const float mn = fmaxf(m, mx);
    const float mref = (mn == -INFINITY) ? 0.f : mn;
    // sum of 2^(x - mref): packed exponent arguments, 8 partial sums
    const float2 ce2 = make_float2(ce, ce), nm2 = make_float2(-mref, -mref);
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int c = 0; c < W; c += 2) {
        const float2 x = ffma2(make_float2(s[C0 + c], s[C0 + c + 1]), ce2, nm2);
        acc[(c >> 1) & 3] = fadd2(acc[(c >> 1) & 3], make_float2(ex2(x.x), ex2(x.y)));
    }
    const float2 t01 = fadd2(acc[0], acc[1]), t23 = fadd2(acc[2], acc[3]);
    const float sum = (t01.x + t01.y) + (t23.x + t23.y);
    L = L * ex2(m - mref) + sum;
    m = mn;
}

// P = 2^(x * ce - mb) over score columns [C0, C0 + W), then those P in the
// storage dtype -> tensor memory, W/2 packed columns from tp + C0/2.
template <typename T, int C0, int W, int N>
__device__ __forceinline__ void p_half(float (&s)[N], float2 ce2, float2 nb2, uint32_t tp) {
#pragma unroll
    for (int c = 0; c < W; c += 2) {
        const float2 x = ffma2(make_float2(s[C0 + c], s[C0 + c + 1]), ce2, nb2);
        s[C0 + c] = ex2(x.x);
        s[C0 + c + 1] = ex2(x.y);
    }
#pragma unroll
    for (int c = 0; c < W / 32; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack2<T>(s[C0 + c * 32 + 2 * e], s[C0 + c * 32 + 2 * e + 1]);
        tmem_st16(tp + C0 / 2 + c * 16, w);
    }
}

template <typename T, int A, bool kMask>
__global__ void __launch_bounds__(kAttnThreads, 1)
nsa_cmp_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    constexpr int NKV = kv_cols_for(A);            // compressed blocks per KV tile
    constexpr int NJ = NKV / A;                    // importance anchors per KV tile
    constexpr int NTAP = 2 * A - 1;                // band taps u = 0 .. 2A-2 (b <= a)
    constexpr int NCARRY = (2 * A - 2) > 0 ? (2 * A - 2) : 1;
    constexpr int ENT = NJ < kEntryMax ? NJ : kEntryMax;   // anchors per staging entry
    constexpr int NENT = NJ / ENT;                 // staging entries per KV tile
    constexpr int STR = ENT + 4;                   // staging row stride in floats
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    static_assert(NJ % ENT == 0 && ENT % 4 == 0, "anchor chunking");

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
        mbar_init(bar(B_Q_FULL0), 1);
        mbar_init(bar(B_Q_FULL1), 1);
        mbar_init(bar(B_Q_EMPTY0), 1);
        mbar_init(bar(B_Q_EMPTY1), 1);
        mbar_init(bar(B_S_FULL0), 1);
        mbar_init(bar(B_S_FULL1), 1);
        mbar_init(bar(B_S_EMPTY0), 4);
        mbar_init(bar(B_S_EMPTY1), 4);
        mbar_init(bar(B_P_FULL), 4);
        mbar_init(bar(B_P_EMPTY), 1);
        mbar_init(bar(B_O_FULL), 1);
        mbar_init(bar(B_O_EMPTY), 4);
        mbar_init(bar(B_STG_FULL0), 4);
        mbar_init(bar(B_STG_FULL1), 4);
        mbar_init(bar(B_STG_EMPTY0), 4);
        mbar_init(bar(B_STG_EMPTY1), 4);
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

    if (warp >= 8) setmaxnreg_dec<kRegsCtl>();
    if (warp == 8) {
        // ============================ TMA producer ============================
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
                const AttnTile t = p.tiles[tile];
                const int qb = tcount % nqbuf;
                const uint32_t qph = (tcount / nqbuf) & 1;
                ok = mbar_wait(bar(B_Q_EMPTY0 + qb), qph ^ 1, abort_flag, p.err, kErrTimeoutBase + 3);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(B_Q_FULL0 + qb), q_bytes);
                const uint32_t qdst = q_addr0 + qb * p.q_bytes;
                for (int c = 0; c < nqc; ++c)
                    tma_load_3d(qdst + c * 16384, &tm_q, c * 64, t.group * G, t.q_row0, bar(B_Q_FULL0 + qb));
                for (int i = 0; i < t.nkv && ok; ++i) load_kv(false, t.group, t.cmp_row0 + i * NKV);
                if (t.nkv > 0 && ok) load_kv(false, t.group, t.cmp_row0);
                for (int i = 0; i < t.nkv && ok; ++i) {
                    if (i + 1 < t.nkv) load_kv(false, t.group, t.cmp_row0 + (i + 1) * NKV);
                    load_kv(true, t.group, t.cmp_row0 + i * NKV);
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
                const AttnTile t = p.tiles[tile];
                const int qb = tcount % nqbuf;
                ok = mbar_wait(bar(B_Q_FULL0 + qb), (tcount / nqbuf) & 1, abort_flag, p.err, kErrTimeoutBase + 6);
                if (!ok) break;
                tc_fence_after();
                q_addr = q_addr0 + qb * p.q_bytes;
                for (int i = 0; i < t.nkv && ok; ++i) issue_s();          // pass A
                if (t.nkv > 0 && ok) issue_s();                          // pass B, S_0
                for (int i = 0; i < t.nkv && ok; ++i) {
                    if (i + 1 < t.nkv) issue_s();
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
                // O_FULL of this tile may only complete after the epilogue of the
                // previous tile has released O: otherwise a tile without PV work
                // could advance O_FULL by two phases before its consumer looks
                if (t.nkv == 0)
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
        // ===================== softmax + band values (128 thr) =====================
        setmaxnreg_inc<kRegsSoftmax>();
        const int row = warp * 32 + lane;          // tile row = TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const int a = p.a, bb = p.b;
        const float c2 = p.scale_log2;
        float wband[NTAP];
#pragma unroll
        for (int u = 0; u < NTAP; ++u) {
            // multiplicity of m + n = u with m < a, n < b (the double sum of step 4)
            const int c = min(min(u, a - 1), min(bb - 1, a + bb - 2 - u)) + 1;
            wband[u] = (u <= a + bb - 2) ? (float)c : 0.f;
        }
        float* stage = reinterpret_cast<float*>(smem + p.off_stage);
        uint32_t scnt = 0, pcnt = 0, stg = 0;
        const int h = row % G;
        const int tok = row / G;

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
        // scores of one KV tile in "exponent units": x = s * ce - shift.  With a
        // positive scale the raw scores are used as they are (ce = c2); a zero
        // or negative scale first multiplies them in (ce = 1).  Columns c >= lim
        // are not visible and become -inf.
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
        // A 128-column score tile is taken in two halves: the second half's
        // tensor-memory load is in flight while the first half is processed.
        // open_half0 waits for the tile, loads columns [0, 64) and starts the
        // load of [64, 128) into r1; close_half1 waits for it and releases the
        // score buffer.  Columns c >= lim are masked as in prep.
        constexpr bool kSplit = (NKV == 128 && A >= 4);   // measured: no gain for a <= 2
        constexpr int NH = kSplit ? NKV / 2 : 16;   // (16: the split helpers are unused then)
        auto mask_half = [&](float (&s)[NKV], int c0, int lim) {
            if (!pos_scale) {
#pragma unroll
                for (int c = 0; c < NH; ++c) s[c0 + c] *= c2;
            }
            if (lim < c0 + NH) {
#pragma unroll
                for (int c = 0; c < NH; ++c) s[c0 + c] = (c0 + c < lim) ? s[c0 + c] : -INFINITY;
            }
        };
        // atten_mask (step 1), masked kernel only: a set byte at (the row's
        // query index, block) removes a visible block.  arow is the row's mask
        // row, null for rows outside the tile or without a mask.
        const uint8_t* arow = nullptr;
        auto amask_cols = [&](float (&s)[NKV], int c0, int w, int i, int lim) {
            if constexpr (kMask) {
                if (arow != nullptr) {
                    const uint8_t* mr = arow + (long long)i * NKV;
#pragma unroll
                    for (int c = 0; c < NKV; ++c)
                        if (c >= c0 && c < c0 + w && c < lim && mr[c]) s[c] = -INFINITY;
                }
            }
        };
        uint32_t split_sb = 0;
        auto open_half0 = [&](float (&s)[NKV], uint32_t (&r1)[NH]) {
            split_sb = scnt % nsbuf;
            mbar_wait(bar(B_S_FULL0 + split_sb), (scnt / nsbuf) & 1, abort_flag, p.err, kErrTimeoutBase + 10);
            tc_fence_after();
            const uint32_t ta = tmem + lane_off + split_sb * 128;
            uint32_t r0[NH];
            tmem_ld_cols<NH>(ta, r0);
            tmem_wait_ld_regs<NH>(r0);
#pragma unroll
            for (int e = 0; e < NH; ++e) s[e] = __uint_as_float(r0[e]);
            tmem_ld_cols<NH>(ta + NH, r1);
        };
        auto close_half1 = [&](float (&s)[NKV], uint32_t (&r1)[NH]) {
            tmem_wait_ld_regs<NH>(r1);
#pragma unroll
            for (int e = 0; e < NH; ++e) s[NH + e] = __uint_as_float(r1[e]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_S_EMPTY0 + split_sb));
            ++scnt;
        };
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

        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
            const AttnTile t = p.tiles[tile];
            const bool valid = (row < TT * G) && (tok < t.ntok);
            const int tpos = t.t0 + tok;
            const int nvis = valid ? nvis_of(tpos, p.l, p.d, t.n_cmp) : 0;
            if constexpr (kMask)
                arow = (valid && p.amask != nullptr) ? p.amask + (long long)(t.tloc0 + tok) * p.am_s2 : nullptr;

            // ---------------- pass A: exact row max and sum (log2 domain) ----------------
            float m = -INFINITY, L = 0.f;
            for (int i = 0; i < t.nkv && kSplit; ++i) {
                float s[NKV];
                uint32_t r1[NH];
                open_half0(s, r1);
                mask_half(s, 0, nvis - i * NKV);
                amask_cols(s, 0, NH, i, nvis - i * NKV);
                online_update<0, NH>(s, ce, m, L);
                close_half1(s, r1);
                mask_half(s, NH, nvis - i * NKV);
                amask_cols(s, NH, NH, i, nvis - i * NKV);
                online_update<NH, NH>(s, ce, m, L);
            }
            for (int i = 0; i < t.nkv && !kSplit; ++i) {
                float s[NKV];
                load_s(s);
                prep(s, nvis - i * NKV);
                amask_cols(s, 0, NKV, i, nvis - i * NKV);
                // row maximum: four independent chains of 3-input max
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
                // row sum of 2^(x - mref): packed exponent arguments, 8 partial sums
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
                const size_t si = ((size_t)(t.q_row0 + tok) * p.n1 + (size_t)t.group * G + h) * 8;
                const float mo = (m == -INFINITY) ? -INFINITY : m * 0.69314718055994530942f;
                const float4 mv = make_float4(mo, mo, mo, mo);
                const float4 lv = make_float4(L, L, L, L);
                reinterpret_cast<float4*>(p.smax + si)[0] = mv;
                reinterpret_cast<float4*>(p.smax + si)[1] = mv;
                reinterpret_cast<float4*>(p.ssum + si)[0] = lv;
                reinterpret_cast<float4*>(p.ssum + si)[1] = lv;
            }

            // ------------- pass B: P -> TMEM, band values -> staging -------------
            // P = 2^(s*c2 - m - log2 L): normalised in the exponent
            const float mb = (L > 0.f) ? m + lg2(L) : INFINITY;
            float carry[NCARRY];
#pragma unroll
            for (int k = 0; k < NCARRY; ++k) carry[k] = 0.f;
            const float2 ce2b = make_float2(ce, ce), nb2 = make_float2(-mb, -mb);
            for (int i = 0; i < t.nkv; ++i) {
                float s[NKV];
                if constexpr (kSplit) {
                    uint32_t r1[NH];
                    open_half0(s, r1);
                    mask_half(s, 0, nvis - i * NKV);
                    amask_cols(s, 0, NH, i, nvis - i * NKV);
                    // P of the previous tile has been read by its P V
                    mbar_wait(bar(B_P_EMPTY), (pcnt & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 11);
                    tc_fence_after();
                    p_half<T, 0, NH>(s, ce2b, nb2, tmem_p + lane_off);
                    close_half1(s, r1);
                    mask_half(s, NH, nvis - i * NKV);
                    amask_cols(s, NH, NH, i, nvis - i * NKV);
                    p_half<T, NH, NH>(s, ce2b, nb2, tmem_p + lane_off);
                } else {
                load_s(s);
                prep(s, nvis - i * NKV);
                amask_cols(s, 0, NKV, i, nvis - i * NKV);
                {
#pragma unroll
                    for (int c = 0; c < NKV; c += 2) {
                        const float2 x = ffma2(make_float2(s[c], s[c + 1]), ce2b, nb2);
                        s[c] = ex2(x.x);
                        s[c + 1] = ex2(x.y);
                    }
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
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_P_FULL));
                ++pcnt;
                // step 4 on the fp32 P: anchors A*jj of this tile; taps reach back
                // into the previous tile through `carry` (carry[k] = P[c0 - 1 - k])
#pragma unroll
                for (int e = 0; e < NENT; ++e) {
                    float v[ENT];
#pragma unroll
                    for (int qq = 0; qq < ENT; ++qq) {
                        const int anchor = A * (e * ENT + qq);
                        float acc = 0.f;
#pragma unroll
                        for (int u = 0; u < NTAP; ++u) {
                            const int x = anchor - u;
                            const float pv = (x >= 0) ? s[x >= 0 ? x : 0] : carry[x < 0 ? (-x - 1) : 0];
                            acc = fmaf(wband[u], pv, acc);
                        }
                        v[qq] = acc;
                    }
                    put_entry(v);
                }
#pragma unroll
                for (int k = 0; k < NCARRY; ++k) carry[k] = s[NKV - 1 - k];
            }
            if (t.nkv > 0) {
                // the first anchors past the last tile still collect taps from it
                float v[ENT];
#pragma unroll
                for (int qq = 0; qq < ENT; ++qq) {
                    const int anchor = A * qq;
                    float acc = 0.f;
#pragma unroll
                    for (int u = 0; u < NTAP; ++u) {
                        const int x = anchor - u;
                        if (x < 0) acc = fmaf(wband[u], carry[-x - 1 >= 0 ? -x - 1 : 0], acc);
                    }
                    v[qq] = acc;
                }
                put_entry(v);
            }
        }
    } else if (warp < 8) {
        // ============ epilogue: group sum, output, top-k (128 thr) ============
        setmaxnreg_dec<kRegsEpilogue>();
        const int ew = warp - 4;                   // TMEM lane quadrant
        const int erow = ew * 32 + lane;
        const int et = threadIdx.x - 128;          // 0..127
        const uint32_t lane_off = (uint32_t)(ew * 32) << 16;
        const float* stage = reinterpret_cast<const float*>(smem + p.off_stage);
        float* score = p.score_in_smem ? reinterpret_cast<float*>(smem + p.off_score)
                                       : p.score_gmem + (size_t)blockIdx.x * TT * p.score_cap;
        const int cap = p.score_cap;
        uint32_t stg = 0;
        int tcount = 0;
        const int eh = erow % G;
        const int etok = erow / G;

        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
            const AttnTile t = p.tiles[tile];
            // step 5: staged band values summed over the G rows of each token
            const int nent = t.nkv > 0 ? t.nkv * NENT + 1 : 0;
            for (int e = 0; e < nent; ++e) {
                const int slot = stg & 1;
                mbar_wait(bar(B_STG_FULL0 + slot), (stg >> 1) & 1, abort_flag, p.err, kErrTimeoutBase + 14);
                const int j0 = (e < t.nkv * NENT) ? (e / NENT) * NJ + (e % NENT) * ENT : t.nkv * NJ;
                const float* st = stage + (size_t)slot * (p.stage_entry_bytes / 4);
                for (int pi = et; pi < t.ntok * ENT; pi += 128) {
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
                    const int j = j0 + jj;
                    if (j < cap) score[tau * cap + j] = (a0 + a1) + (a2 + a3);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_STG_EMPTY0 + slot));
                ++stg;
            }
            const int jcov = t.nkv > 0 ? t.nkv * NJ + ENT : 0;

            // O (tensor memory) -> attention_out
            mbar_wait(bar(B_O_FULL), tcount & 1, abort_flag, p.err, kErrTimeoutBase + 12);
            tc_fence_after();
            {
                const bool valid = (erow < TT * G) && (etok < t.ntok);
                const int nvis = valid ? nvis_of(t.t0 + etok, p.l, p.d, t.n_cmp) : 0;
                T* orow = reinterpret_cast<T*>(p.out) +
                          ((size_t)(t.q_row0 + etok) * p.n1 + (size_t)t.group * G + eh) * p.d2;
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

            named_bar_sync(2, 128);   // every group sum of this tile is in the score buffer
            // step 7, one warp per token
            for (int tau = ew; tau < t.ntok; tau += 4) {
                const int tp = t.t0 + tau;
                int32_t* dst = p.topk + ((size_t)(t.q_row0 + tau) * p.n2 + t.group) * p.count;
                const int nv = nvis_of(tp, p.l, p.d, t.n_cmp);
                bool empty = nv == 0;
                const uint8_t* trow = nullptr;
                if constexpr (kMask) {
                    // a token whose visible blocks are all masked attends to nothing
                    if (!empty && p.amask != nullptr) {
                        const uint8_t* ar = p.amask + (long long)(t.tloc0 + tau) * p.am_s2;
                        int keep = 0;
                        for (int c = lane; c < nv; c += 32) keep |= (ar[c] == 0) ? 1 : 0;
                        empty = !__any_sync(0xffffffffu, keep);
                    }
                    if (p.tmask != nullptr) trow = p.tmask + (long long)(t.tloc0 + tau) * p.tm_s2;
                }
                if (empty) {
                    for (int j = lane; j < p.count; j += 32) dst[j] = -1;
                } else {
                    const int ncand = min(t.n_sel, tp / p.lp + 1);
                    warp_topk<kMask>(score + tau * cap, ncand, jcov, p.count, dst, lane, trow);
                }
            }
            named_bar_sync(2, 128);   // the score buffer is free for the next tile
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

template <typename T, int A, bool kMask>
static cudaError_t launch_t(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, int grid, cudaStream_t st) {
    auto kern = nsa_cmp_attn_kernel<T, A, kMask>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kAttnThreads, p.smem_bytes, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

template <typename T, bool kMask>
static cudaError_t launch_a(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, int grid, cudaStream_t st) {
    switch (p.a) {
        case 1: return launch_t<T, 1, kMask>(p, tq, tk, tv, grid, st);
        case 2: return launch_t<T, 2, kMask>(p, tq, tk, tv, grid, st);
        case 3: return launch_t<T, 3, kMask>(p, tq, tk, tv, grid, st);
        case 4: return launch_t<T, 4, kMask>(p, tq, tk, tv, grid, st);
        case 5: return launch_t<T, 5, kMask>(p, tq, tk, tv, grid, st);
        case 6: return launch_t<T, 6, kMask>(p, tq, tk, tv, grid, st);
        case 7: return launch_t<T, 7, kMask>(p, tq, tk, tv, grid, st);
        case 8: return launch_t<T, 8, kMask>(p, tq, tk, tv, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_attention(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, int grid, cudaStream_t st) {
    // the masked kernel only where a mask is given: the unmasked one is unchanged
    if (p.amask != nullptr || p.tmask != nullptr)
        return p.dtype == 0 ? launch_a<__nv_bfloat16, true>(p, tq, tk, tv, grid, st)
                            : launch_a<__half, true>(p, tq, tk, tv, grid, st);
    return p.dtype == 0 ? launch_a<__nv_bfloat16, false>(p, tq, tk, tv, grid, st)
                        : launch_a<__half, false>(p, tq, tk, tv, grid, st);
}

}  // namespace nsa
