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
// one KV group), so every row of the tile shares one K/V head and the group
// sum of step 5 is a sum over neighbouring rows.  Per tile, two passes over
// the compressed keys (the importance scores sum *normalised* probabilities
// over heads, and a head's normaliser is only known at the end of its row):
//   pass A  S = Q K^T on the tensor cores (tcgen05.mma, fp32 in TMEM),
//           online max / sum in registers -> exact m and L per row.
//   pass B  S = Q K^T again, P = exp(S - m) / L in fp32 registers, bf16/fp16 P
//           -> shared memory -> O += P V on the tensor cores; from the fp32 P
//           the banded importance sum (step 4) and the group sum (step 5) go
//           to a per-token score buffer that never leaves the SM.
//   epilogue O (TMEM) -> out; stats; radix-select top-k per token (step 7).
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 issues the MMAs
// and owns the tensor memory, warps 2-5 (one thread per tile row, matching
// the four 32-lane quadrants of TMEM) run softmax, band sums and epilogue.
// Q, K and V are staged by TMA with 128-byte swizzle; K/V share one ring.
// Every mbarrier wait is bounded; a timeout sets the workspace error word.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cfloat>
#include <type_traits>

#include "nsa_internal.h"
#include "ptx.cuh"

namespace nsa {

__host__ __device__ constexpr int kv_cols_for(int a) {
    // largest multiple of lcm(16, a) not above 128: every KV tile then holds a
    // whole number of importance anchors (anchor of block j = a*j)
    return (a == 1 || a == 2 || a == 4 || a == 8) ? 128
           : (a == 3 || a == 6)                   ? 96
           : (a == 5)                             ? 80
                                                  : 112;
}

int attention_kv_cols(int a) { return kv_cols_for(a); }

enum BarId {
    B_Q_FULL = 0,
    B_Q_EMPTY,
    B_S_FULL0,
    B_S_FULL1,
    B_S_EMPTY0,
    B_S_EMPTY1,
    B_P_FULL,
    B_P_EMPTY,
    B_O_FULL,
    B_O_EMPTY,
    B_MMA_DONE,
    B_SLOT_FULL0,            // + slot
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
// Exact k-th largest key by a bitwise search over the fp32 bit patterns
// (scores are >= 0, so the bit patterns order like the values), then an
// ordered ballot scan keeps every key above it plus the earliest ties.
__device__ __forceinline__ void warp_topk(const float* sc, int ncand, int jcov, int count,
                                          int32_t* dst, int lane) {
    const int k = min(count, ncand);
    if (k == ncand) {
        for (int j = lane; j < count; j += 32) dst[j] = (j < ncand) ? j : -1;
        return;
    }
    auto key = [&](int j) -> uint32_t { return j < jcov ? __float_as_uint(sc[j]) : 0u; };
    uint32_t thr = 0;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t trial = thr | (1u << bit);
        int c = 0;
        for (int j = lane; j < ncand; j += 32) c += key(j) >= trial ? 1 : 0;
        c = __reduce_add_sync(0xffffffffu, c);
        if (c >= k) thr = trial;
    }
    int ngt = 0;
    for (int j = lane; j < ncand; j += 32) ngt += key(j) > thr ? 1 : 0;
    ngt = __reduce_add_sync(0xffffffffu, ngt);
    const int need_eq = k - ngt;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int eq_seen = 0, written = 0;
    for (int base = 0; base < ncand; base += 32) {
        const int j = base + lane;
        const bool in = j < ncand;
        const uint32_t kv = in ? key(j) : 0u;
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

template <typename T, int A>
__global__ void __launch_bounds__(kAttnThreads, 1)
nsa_cmp_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    constexpr int NKV = kv_cols_for(A);            // compressed blocks per KV tile
    constexpr int NJ = NKV / A;                    // importance anchors per KV tile
    constexpr int NTAP = 2 * A - 1;                // band taps u = 0 .. 2A-2 (b <= a)
    constexpr int NCARRY = (2 * A - 2) > 0 ? (2 * A - 2) : 1;
    constexpr int CHK = NJ < kBandChunk ? NJ : kBandChunk;
    constexpr int STG = CHK + 1;                   // staging row stride (odd: no bank conflicts)
    constexpr bool kBF16 = sizeof(T) == 2 && std::is_same<T, __nv_bfloat16>::value;
    static_assert(NJ % CHK == 0, "anchor chunking");

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
        mbar_init(bar(B_Q_FULL), 1);
        mbar_init(bar(B_Q_EMPTY), 1);
        mbar_init(bar(B_S_FULL0), 1);
        mbar_init(bar(B_S_FULL1), 1);
        mbar_init(bar(B_S_EMPTY0), 4);
        mbar_init(bar(B_S_EMPTY1), 4);
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
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + 256;

    const uint32_t q_addr = smem_u32(smem + p.off_q);
    const uint32_t ring_addr = smem_u32(smem + p.off_ring);
    const uint32_t p_addr = smem_u32(smem + p.off_p);
    const int nslot = p.nslot;
    const int nqc = (p.d1 + 63) / 64;    // 64-element chunks of a Q/K row
    const int nvc = (p.d2 + 63) / 64;    // 64-element chunks of a V row

    if (warp == 0) {
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
                ok = mbar_wait(bar(B_Q_EMPTY), (tcount & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 3);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(B_Q_FULL), q_bytes);
                for (int c = 0; c < nqc; ++c)
                    tma_load_3d(q_addr + c * 16384, &tm_q, c * 64, t.group * G, t.q_row0, bar(B_Q_FULL));
                for (int i = 0; i < t.nkv && ok; ++i) load_kv(false, t.group, t.cmp_row0 + i * NKV);
                if (t.nkv > 0 && ok) load_kv(false, t.group, t.cmp_row0);
                for (int i = 0; i < t.nkv && ok; ++i) {
                    if (i + 1 < t.nkv) load_kv(false, t.group, t.cmp_row0 + (i + 1) * NKV);
                    load_kv(true, t.group, t.cmp_row0 + i * NKV);
                }
            }
        }
    } else if (warp == 1) {
        // ============================ MMA issuer =============================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_f16(kBF16, 128, NKV, false, false);
            const uint32_t idesc_pv = idesc_f16(kBF16, 128, p.d2, false, true);
            const int nks_qk = p.d1 / 16;
            constexpr int nks_pv = NKV / 16;
            uint32_t item = 0, scnt = 0, pcnt = 0;
            int tcount = 0;
            bool ok = true;
            auto issue_s = [&]() {
                const int sb = scnt & 1;
                ok = ok && mbar_wait(bar(B_S_EMPTY0 + sb), ((scnt >> 1) & 1) ^ 1, abort_flag, p.err,
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
                ok = mbar_wait(bar(B_Q_FULL), tcount & 1, abort_flag, p.err, kErrTimeoutBase + 6);
                if (!ok) break;
                tc_fence_after();
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
                        const uint64_t ad = sdesc_sw128(p_addr + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(vbase + ks * 2048, NKV * 128, 1024);
                        umma_ss(tmem_o, ad, bd, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
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
                umma_commit(bar(B_Q_EMPTY));
            }
            // every MMA issued so far has retired before the tensor memory is freed
            umma_commit(bar(B_MMA_DONE));
            mbar_wait(bar(B_MMA_DONE), 0, abort_flag, nullptr, 0);
        }
    } else {
        // ==================== softmax / band / epilogue (128 thr) ====================
        const int wq = warp & 3;                  // TMEM lane quadrant of this warp
        const int row = wq * 32 + lane;           // tile row = TMEM lane
        const int st = threadIdx.x - 64;          // 0..127, for row-independent work
        const int sw = warp - 2;                  // 0..3
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const int a = p.a, bb = p.b;
        float wband[NTAP];
#pragma unroll
        for (int u = 0; u < NTAP; ++u) {
            // multiplicity of m + n = u with m < a, n < b (step 4 double sum)
            const int c = min(min(u, a - 1), min(bb - 1, a + bb - 2 - u)) + 1;
            wband[u] = (u <= a + bb - 2) ? (float)c : 0.f;
        }
        float* stage = reinterpret_cast<float*>(smem + p.off_stage);
        float* score = p.score_in_smem ? reinterpret_cast<float*>(smem + p.off_score)
                                       : p.score_gmem + (size_t)blockIdx.x * TT * p.score_cap;
        const int cap = p.score_cap;
        uint32_t scnt = 0, pcnt = 0;
        int tcount = 0;
        const int h = row % G;
        const int tok = row / G;

        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
            const AttnTile t = p.tiles[tile];
            const bool valid = (row < TT * G) && (tok < t.ntok);
            const int tpos = t.t0 + tok;
            const int nvis = valid ? nvis_of(tpos, p.l, p.d, t.n_cmp) : 0;

            auto load_s = [&](float (&s)[NKV]) {
                const int sb = scnt & 1;
                mbar_wait(bar(B_S_FULL0 + sb), (scnt >> 1) & 1, abort_flag, p.err, kErrTimeoutBase + 10);
                tc_fence_after();
                const uint32_t ta = tmem + lane_off + sb * 128;
#pragma unroll
                for (int c = 0; c < NKV / 16; ++c) {
                    uint32_t r[16];
                    tmem_ld16(ta + c * 16, r);
#pragma unroll
                    for (int e = 0; e < 16; ++e) s[c * 16 + e] = __uint_as_float(r[e]);
                }
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_S_EMPTY0 + sb));
                ++scnt;
            };

            // ---------------- pass A: exact row max and sum ----------------
            float m = -INFINITY, L = 0.f;
            for (int i = 0; i < t.nkv; ++i) {
                float s[NKV];
                load_s(s);
                const int lim = nvis - i * NKV;     // columns c < lim are visible
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < NKV; ++c) {
                    s[c] = (c < lim) ? s[c] * p.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, s[c]);
                }
                const float mn = fmaxf(m, mx);
                const float mref = (mn == -INFINITY) ? 0.f : mn;
                float sum = 0.f;
#pragma unroll
                for (int c = 0; c < NKV; ++c) sum += ex2(s[c] - mref);
                L = L * ex2(m - mref) + sum;
                m = mn;
            }

            // ------------- pass B: P, PV, importance band, group sum -------------
            const float invL = (L > 0.f) ? 1.f / L : 0.f;
            const float mref = (m == -INFINITY) ? 0.f : m;
            float carry[NCARRY];
#pragma unroll
            for (int k = 0; k < NCARRY; ++k) carry[k] = 0.f;

            // stage CHK anchors per round, reduce over the G rows of each token
            auto band_round = [&](const float* vals, int jfirst) {
#pragma unroll
                for (int qq = 0; qq < CHK; ++qq) stage[row * STG + qq] = vals[qq];
                named_bar_sync(1, 128);
                for (int pi = st; pi < t.ntok * CHK; pi += 128) {
                    const int tau = pi / CHK, qq = pi - tau * CHK;
                    const float* src = stage + (tau * G) * STG + qq;
                    float acc = 0.f;
                    for (int hh = 0; hh < G; ++hh) acc += src[hh * STG];
                    const int j = jfirst + qq;
                    if (j < cap) score[tau * cap + j] = acc;
                }
                named_bar_sync(1, 128);
            };

            for (int i = 0; i < t.nkv; ++i) {
                float s[NKV];
                load_s(s);
                const int lim = nvis - i * NKV;
#pragma unroll
                for (int c = 0; c < NKV; ++c)
                    s[c] = (c < lim) ? ex2(s[c] * p.scale_log2 - mref) * invL : 0.f;
                // P (storage dtype) -> shared memory, K-major, 128-byte swizzle
                mbar_wait(bar(B_P_EMPTY), (pcnt & 1) ^ 1, abort_flag, p.err, kErrTimeoutBase + 11);
                {
                    uint8_t* prow = smem + p.off_p + row * 128;
#pragma unroll
                    for (int v = 0; v < NKV / 8; ++v) {
                        const int chunk = v >> 3, unit = v & 7;
                        uint4 w;
                        w.x = pack2<T>(s[v * 8 + 0], s[v * 8 + 1]);
                        w.y = pack2<T>(s[v * 8 + 2], s[v * 8 + 3]);
                        w.z = pack2<T>(s[v * 8 + 4], s[v * 8 + 5]);
                        w.w = pack2<T>(s[v * 8 + 6], s[v * 8 + 7]);
                        *reinterpret_cast<uint4*>(prow + chunk * 16384 + ((unit ^ (row & 7)) << 4)) = w;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_P_FULL));
                ++pcnt;
                // step 4 on the fp32 P: anchors a*jj of this tile, taps reach back
                // into the previous tile through `carry` (carry[k] = P[c0 - 1 - k])
#pragma unroll
                for (int jc = 0; jc < NJ; jc += CHK) {
                    float vals[CHK];
#pragma unroll
                    for (int qq = 0; qq < CHK; ++qq) {
                        const int anchor = A * (jc + qq);
                        float acc = 0.f;
#pragma unroll
                        for (int u = 0; u < NTAP; ++u) {
                            const int x = anchor - u;
                            const float pv = (x >= 0) ? s[x >= 0 ? x : 0] : carry[x < 0 ? (-x - 1) : 0];
                            acc = fmaf(wband[u], pv, acc);
                        }
                        vals[qq] = acc;
                    }
                    band_round(vals, i * NJ + jc);
                }
#pragma unroll
                for (int k = 0; k < NCARRY; ++k) carry[k] = (NKV - 1 - k >= 0) ? s[NKV - 1 - k] : 0.f;
            }
            int jcov = 0;
            if (t.nkv > 0) {
                // the first anchors past the last tile still collect taps from it
                float vals[CHK];
#pragma unroll
                for (int qq = 0; qq < CHK; ++qq) {
                    const int anchor = A * qq;
                    float acc = 0.f;
#pragma unroll
                    for (int u = 0; u < NTAP; ++u) {
                        const int x = anchor - u;
                        if (x < 0) acc = fmaf(wband[u], carry[-x - 1 >= 0 ? -x - 1 : 0], acc);
                    }
                    vals[qq] = acc;
                }
                band_round(vals, t.nkv * NJ);
                jcov = t.nkv * NJ + CHK;
            }

            // ---------------------------- epilogue ----------------------------
            mbar_wait(bar(B_O_FULL), tcount & 1, abort_flag, p.err, kErrTimeoutBase + 12);
            tc_fence_after();
            {
                T* orow = reinterpret_cast<T*>(p.out) +
                          ((size_t)(t.q_row0 + tok) * p.n1 + (size_t)t.group * G + h) * p.d2;
                for (int c = 0; c < p.d2 / 16; ++c) {
                    uint32_t r[16];
                    tmem_ld16(tmem_o + lane_off + c * 16, r);
                    tmem_wait_ld();
                    if (valid) {
                        uint4 w0, w1;
                        float f[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) f[e] = (nvis > 0) ? __uint_as_float(r[e]) : 0.f;
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
            // step 7, one warp per token
            for (int tau = sw; tau < t.ntok; tau += 4) {
                const int tp = t.t0 + tau;
                int32_t* dst = p.topk + ((size_t)(t.q_row0 + tau) * p.n2 + t.group) * p.count;
                if (nvis_of(tp, p.l, p.d, t.n_cmp) == 0) {
                    for (int j = lane; j < p.count; j += 32) dst[j] = -1;
                } else {
                    const int ncand = min(t.n_sel, tp / p.lp + 1);
                    warp_topk(score + tau * cap, ncand, jcov, p.count, dst, lane);
                }
            }
            named_bar_sync(1, 128);   // score buffer is free for the next tile
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
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <typename T, int A>
static cudaError_t launch_t(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, int grid, cudaStream_t st) {
    auto kern = nsa_cmp_attn_kernel<T, A>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
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

cudaError_t launch_attention(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, int grid, cudaStream_t st) {
    return p.dtype == 0 ? launch_a<__nv_bfloat16>(p, tq, tk, tv, grid, st)
                        : launch_a<__half>(p, tq, tk, tv, grid, st);
}

}  // namespace nsa
