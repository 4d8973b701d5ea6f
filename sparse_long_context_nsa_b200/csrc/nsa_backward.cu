// nsa_backward.cu -- gradients of compressed attention and of the compression
// (sm_100a).
//
// The pages return softmax_max / softmax_sum "for gradient backprop"
// ("mindspore.ops.nsa_compress_attention", Returns list; the softmax_lse of
// "lite_boost.ops.rain_fusion_attention") and place the compression in the
// training scenario ("aclnnNsaCompress", operator description), but print no
// backward formulas.  They follow from the forward definition (steps 1-3; the
// importance scores and the top-k are index outputs and carry no gradient):
//   P_i  = exp(s_i - m) / L,  s_i = scale q . kcmp_i   (visible blocks)
//   dV_i = sum over rows of P_i dout           (summed over the G heads of a group)
//   dP_i = dout . vcmp_i,  delta = sum_i P_i dP_i = dout . out
//   dS_i = P_i (dP_i - delta)
//   dq   = scale sum_i dS_i kcmp_i,   dK_i = scale sum over rows of dS_i q
// and for the compression kcmp_i = sum_j w_j k[i d + j] (linear):
//   dk[p] = sum_i w[p - i d] dkcmp_i,   dw_j = sum_i dkcmp_i . k[i d + j]  (+ the V terms).
//
// Kernels:
//   prep     per (row, head): delta = out . dout and the log2 normaliser
//            m log2e + log2 L from the saved statistics.
//   dq       one query M-tile (TT tokens x G heads) over its visible KV tiles
//            of 128 blocks: S = Q K^T and dP = dO V^T by tcgen05.mma into
//            tensor memory; the softmax warps (one row each) write dS in the
//            storage dtype over S; dQ += dS K with dS read from tensor memory.
//   dkdv     one KV tile of one group over the query M-tiles that see it, in
//            halves of 64 rows: S^T = K Q^T and dP^T = V dO^T; P^T and dS^T
//            over them; dV += P^T dO and dK += dS^T Q.  The rows of an M-tile
//            are the G heads of the group, so the sums over the heads come out
//            of the contraction.  Each tile's dK, dV are written once: no
//            atomics, deterministic.
//   dx / dw  the compression transposed: dk / dv gathered per raw row from the
//            windows that cover it; dw reduced per (window position, head) over
//            every compressed row in a fixed order.
// One work item per CTA, the MMA steps issued in order and waited for (a first
// form, correct before fast).  Every mbarrier wait is bounded and reports a
// timeout in the workspace error word.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <type_traits>

#include "nsa_internal.h"
#include "ptx.cuh"

namespace nsa {
namespace bwd {

template <typename T>
__device__ __forceinline__ uint32_t pk2(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pk2<__nv_bfloat16>(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pk2<__half>(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
template <typename T>
__device__ __forceinline__ float2 up2(uint32_t w);
template <>
__device__ __forceinline__ float2 up2<__nv_bfloat16>(uint32_t w) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w));
}
template <>
__device__ __forceinline__ float2 up2<__half>(uint32_t w) {
    return __half22float2(*reinterpret_cast<__half2*>(&w));
}

__device__ __forceinline__ int nvis_at(int t, int l, int d, int n_cmp) {
    // compressed block i is visible to position t iff i*d + l - 1 <= t
    if (t < l - 1) return 0;
    return min(n_cmp, (t - l + 1) / d + 1);
}

// B_Q0/1 and B_KV0/1: one barrier per stage of the two-stage rings; B_S0/1, B_P0/1: one per
// score buffer; B_QE0/1: a Q/dO stage's last reader has retired
enum Bar { B_Q0 = 0, B_Q1, B_KV0, B_KV1, B_S0, B_S1, B_P0, B_P1, B_QE0, B_QE1, B_MMA, B_DONE, B_N };

// ------------------------------------------------------------------- prep
// One warp per row: delta = sum_e out * dout (fp32) and the row's log2
// normaliser; rows that attended to nothing (L = 0) get +inf, so P = 0.
template <typename T>
__global__ void prep_kernel(const T* __restrict__ out, const T* __restrict__ dout, const float* __restrict__ smax,
                            const float* __restrict__ ssum, float2* __restrict__ rowinfo, long long rows, int d2) {
    const int lane = threadIdx.x & 31;
    const long long w0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long r = w0; r < rows; r += nw) {
        float acc = 0.f;
        for (int e = lane * 8; e < d2; e += 256) {
            const uint4 ov = *reinterpret_cast<const uint4*>(out + r * d2 + e);
            const uint4 gv = *reinterpret_cast<const uint4*>(dout + r * d2 + e);
            const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 a = up2<T>(ow[k]), b = up2<T>(gw[k]);
                acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
            const float m = smax[r * 8], L = ssum[r * 8];
            const float mb = (L > 0.f && m > -INFINITY) ? m * 1.4426950408889634f + log2f(L) : INFINITY;
            rowinfo[r] = make_float2(mb, acc);
        }
    }
}

cudaError_t launch_prep(const void* out, const void* dout, const float* smax, const float* ssum, float2* rowinfo,
                        long long rows, int d2, int dtype, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const int threads = 256;   // eight rows at a time per CTA
    const int blocks = (int)std::min<long long>((rows + 7) / 8, 148LL * 16);
    if (dtype == 0)
        prep_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(out), reinterpret_cast<const __nv_bfloat16*>(dout), smax, ssum,
            rowinfo, rows, d2);
    else
        prep_kernel<__half><<<blocks, threads, 0, st>>>(reinterpret_cast<const __half*>(out),
                                                        reinterpret_cast<const __half*>(dout), smax, ssum, rowinfo,
                                                        rows, d2);
    return cudaGetLastError();
}

// --------------------------------------------------------------- shared
struct Smem {
    uint8_t* base;
    uint64_t* bars;
    uint32_t* tmem_slot;
    volatile int* abort_flag;
};

__device__ __forceinline__ Smem smem_setup(const Params& p) {
    extern __shared__ uint8_t smem_raw[];
    Smem s;
    s.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    s.bars = reinterpret_cast<uint64_t*>(s.base + p.off_bar);
    s.tmem_slot = reinterpret_cast<uint32_t*>(s.base + p.off_bar + 8 * B_N);
    s.abort_flag = reinterpret_cast<volatile int*>(s.base + p.off_bar + 8 * B_N + 4);
    return s;
}

// 128 rows x 16 fp32 columns of this warp's lanes -> fp32 global row (x mul)
__device__ __forceinline__ void store_row_f32(uint32_t taddr, int ncols, float mul, float* dst, bool valid) {
    for (int c = 0; c < ncols; c += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + c, r);
        tmem_wait_ld_regs<16>(r);
        if (valid) {
            float4* d4 = reinterpret_cast<float4*>(dst + c);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                d4[q] = make_float4(__uint_as_float(r[4 * q]) * mul, __uint_as_float(r[4 * q + 1]) * mul,
                                    __uint_as_float(r[4 * q + 2]) * mul, __uint_as_float(r[4 * q + 3]) * mul);
        }
    }
}

// --------------------------------------------------------------------- dQ
template <typename T>
__global__ void __launch_bounds__(kThreadsDq, 1)
dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
          const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const Params p) {
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    Smem sm = smem_setup(p);
    auto bar = [&](int id) { return smem_u32(&sm.bars[id]); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const QItem it = p.qitems[blockIdx.x];
    const int G = p.G, TT = p.tok_per_tile;
    const int nqc = (p.d1 + 63) / 64, nvc = (p.d2 + 63) / 64;

    if (threadIdx.x == 0) {
        // dS of a tile is written by eight warps (two per lane quadrant, one per column half)
        for (int i = 0; i < B_N; ++i) mbar_init(bar(i), (i == B_P0 || i == B_P1) ? 8 : 1);
        *sm.abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 4) {
        tmem_alloc(smem_u32(sm.tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sm.tmem_slot;   // S at 0, dP at 128, dQ at 256
    const uint32_t qa = smem_u32(sm.base + p.off_q), doa = smem_u32(sm.base + p.off_do);
    const uint32_t ka = smem_u32(sm.base + p.off_k), va = smem_u32(sm.base + p.off_v);

    if (warp == 4) {
        if (lane == 0) {
            const uint32_t qbytes = nqc * 64 * G * TT * 2, dobytes = nvc * 64 * G * TT * 2;
            const uint32_t kbytes = nqc * 64 * kKV * 2, vbytes = nvc * 64 * kKV * 2;
            constexpr uint32_t id_s = idesc_f16(kBF16, 128, kKV, false, false);
            const uint32_t id_q = idesc_f16(kBF16, 128, p.d1, false, true);
            bool ok = true;
            mbar_arrive_expect_tx(bar(B_Q0), qbytes + dobytes);
            for (int c = 0; c < nqc; ++c)
                tma_load_3d(qa + c * 16384, &tm_q, c * 64, it.group * G, it.q_row0, bar(B_Q0));
            for (int c = 0; c < nvc; ++c)
                tma_load_3d(doa + c * 16384, &tm_do, c * 64, it.group * G, it.q_row0, bar(B_Q0));
            // K/V tiles through a ring of p.nst stages: with two, tile i + 1 loads while
            // tile i computes (its stage was last read by tile i - 1, retired below)
            auto load_kv = [&](int i) {
                const int st = i % p.nst;
                const uint32_t ks0 = ka + st * p.stage_bytes, vs0 = va + st * p.stage_bytes;
                const int row = it.cmp_row0 + i * kKV;
                mbar_arrive_expect_tx(bar(B_KV0 + st), kbytes + vbytes);
                for (int c = 0; c < nqc; ++c) tma_load_3d(ks0 + c * 16384, &tm_k, c * 64, it.group, row, bar(B_KV0 + st));
                for (int c = 0; c < nvc; ++c) tma_load_3d(vs0 + c * 16384, &tm_v, c * 64, it.group, row, bar(B_KV0 + st));
            };
            if (it.nkv > 0) load_kv(0);
            for (int i = 0; i < it.nkv && ok; ++i) {
                const int st = i % p.nst;
                const uint32_t kst = ka + st * p.stage_bytes, vst = va + st * p.stage_bytes;
                ok = mbar_wait(bar(B_KV0 + st), (i / p.nst) & 1, sm.abort_flag, p.err, kErrTimeoutBase + 0x21);
                if (i == 0) ok = ok && mbar_wait(bar(B_Q0), 0, sm.abort_flag, p.err, kErrTimeoutBase + 0x22);
                if (!ok) break;
                if (p.nst == 2 && i + 1 < it.nkv) load_kv(i + 1);
                tc_fence_after();
                for (int ks = 0; ks < p.d1 / 16; ++ks) {   // S = Q K^T
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma_ss(tmem, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(kst + off, 16, 1024), id_s,
                            ks > 0 ? 1u : 0u);
                }
                for (int ks = 0; ks < p.d2 / 16; ++ks) {   // dP = dO V^T
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma_ss(tmem + 128, sdesc_sw128(doa + off, 16, 1024), sdesc_sw128(vst + off, 16, 1024), id_s,
                            ks > 0 ? 1u : 0u);
                }
                umma_commit(bar(B_S0));
                ok = mbar_wait(bar(B_P0), i & 1, sm.abort_flag, p.err, kErrTimeoutBase + 0x23);
                if (!ok) break;
                tc_fence_after();
                for (int ks = 0; ks < kKV / 16; ++ks)   // dQ += dS K (dS from tensor memory: each
                                                        // half of the keys at the start of its half)
                    umma_ts(tmem + 256, tmem + ks * 8 + (ks >= kKV / 32 ? kKV / 4 : 0),
                            sdesc_sw128(kst + ks * 2048, kKV * 128, 1024), id_q, (i > 0 || ks > 0) ? 1u : 0u);
                umma_commit(bar(B_MMA));
                ok = mbar_wait(bar(B_MMA), i & 1, sm.abort_flag, p.err, kErrTimeoutBase + 0x24);
                if (ok && p.nst == 1 && i + 1 < it.nkv) load_kv(i + 1);
            }
        }
    } else {
        // one query row per thread; warps 0-3 take the first half of a tile's columns
        // (and of dQ), warps 5-8 the second, each in its lane quadrant (warp % 4)
        const int quad = warp & 3, half = warp > 4 ? 1 : 0;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int tok = row / G, h = row % G;
        const bool valid = row < TT * G && tok < it.ntok && nsa_index_ok(it.q_row0 + tok < p.rows_q, p.err, 8);
        const int nv = valid ? nvis_at(it.t0 + tok, p.l, p.d, it.n_cmp) : 0;
        const size_t ri = ((size_t)(it.q_row0 + tok) * p.n1 + (size_t)it.group * G + h);
        const float2 info = valid ? p.rowinfo[ri] : make_float2(INFINITY, 0.f);
        const float c2 = p.scale_log2;
        for (int i = 0; i < it.nkv; ++i) {
            mbar_wait(bar(B_S0), i & 1, sm.abort_flag, p.err, kErrTimeoutBase + 0x25);
            tc_fence_after();
#pragma unroll 1
            for (int c = half * (kKV / 64); c < (half + 1) * (kKV / 64); ++c) {
                uint32_t rs[32], rp[32];
                tmem_ld32(tmem + lane_off + c * 32, rs);
                tmem_ld32(tmem + lane_off + 128 + c * 32, rp);
                tmem_wait_ld_regs<32>(rs);
                tmem_wait_ld_regs<32>(rp);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int kb = i * kKV + c * 32 + e;
                    const bool v0 = kb < nv, v1 = kb + 1 < nv;
                    const float p0 = v0 ? ex2(__uint_as_float(rs[e]) * c2 - info.x) : 0.f;
                    const float p1 = v1 ? ex2(__uint_as_float(rs[e + 1]) * c2 - info.x) : 0.f;
                    pk[e >> 1] = pk2<T>(v0 ? p0 * (__uint_as_float(rp[e]) - info.y) : 0.f,
                                        v1 ? p1 * (__uint_as_float(rp[e + 1]) - info.y) : 0.f);
                }
                // dS of the chunk over S columns this warp has already read: the first 32
                // columns of its own half (the other half's warp still reads its S)
                tmem_st16(tmem + lane_off + c * 16 + half * (kKV / 4), pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_P0));
        }
        // this warp's half of the row of dQ (16-column pieces)
        const int c16 = (p.d1 / 16 + 1) / 2;
        const int e0 = half * c16 * 16, e1 = min(p.d1, (half + 1) * c16 * 16);
        float* dst = p.dq + ri * p.d1;
        if (it.nkv > 0) {
            mbar_wait(bar(B_MMA), (it.nkv - 1) & 1, sm.abort_flag, p.err, kErrTimeoutBase + 0x26);
            tc_fence_after();
            if (e1 > e0) store_row_f32(tmem + lane_off + 256 + e0, e1 - e0, p.scale, dst + e0, valid);
        } else if (valid) {
            for (int e = e0; e < e1; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*sm.abort_flag && threadIdx.x == 0) {
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 20000000ull) {
        }
    }
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ dK, dV
// Query rows are the contraction dimension of dV += P^T dO and dK += dS^T Q,
// so every row that takes part must hold finite values: rows of the box past
// G x TT are zeroed once, rows outside the run get P = dS = 0 by selection.
template <typename T>
__global__ void __launch_bounds__(kThreadsDq, 1)
dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const Params p) {
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    Smem sm = smem_setup(p);
    auto bar = [&](int id) { return smem_u32(&sm.bars[id]); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KVItem it = p.kvitems[blockIdx.x];
    const int G = p.G, TT = p.tok_per_tile;
    const int nqc = (p.d1 + 63) / 64, nvc = (p.d2 + 63) / 64;
    const bool do_dv = p.mode & 1, do_dk = (p.mode >> 1) & 1;
    const int n_mt = (it.q_end - it.q_row0 + TT - 1) / TT;   // query M-tiles of the run

    if (threadIdx.x == 0) {
        // Pᵀ and dSᵀ of a step are written by eight warps (two per lane quadrant)
        for (int i = 0; i < B_N; ++i) mbar_init(bar(i), (i == B_P0 || i == B_P1) ? 8 : 1);
        *sm.abort_flag = 0;
        fence_mbar_init();
    }
    {
        // rows G*TT..127 of every Q / dO chunk of every stage: never written by the copies
        const int r0 = G * TT;
        const int nch = nqc + nvc;
        const int per = (128 - r0) * 8;   // 16-byte pieces per chunk
        for (int x = threadIdx.x; x < p.nst * nch * per; x += blockDim.x) {
            const int sc = x / per, o = x % per;
            const int st = sc / nch, c = sc % nch;
            uint8_t* base = sm.base + st * p.stage_bytes +
                            (c < nqc ? p.off_q + c * 16384 : p.off_do + (c - nqc) * 16384);
            *reinterpret_cast<uint4*>(base + r0 * 128 + o * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    if (warp == 4) {
        tmem_alloc(smem_u32(sm.tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sm.tmem_slot;   // dV at 0, dK at col_dk, S^T at 384, dP^T at 448
    const uint32_t qa = smem_u32(sm.base + p.off_q), doa = smem_u32(sm.base + p.off_do);
    const uint32_t ka = smem_u32(sm.base + p.off_k), va = smem_u32(sm.base + p.off_v);
    // the rows' statistics and visible counts, one buffer per M-tile parity
    float2* rinfo2 = reinterpret_cast<float2*>(sm.base + p.off_row);
    int* rnv2 = reinterpret_cast<int*>(sm.base + p.off_row + 2 * 128 * sizeof(float2));

    if (warp == 4) {
        if (lane == 0) {
            const uint32_t qbytes = nqc * 64 * G * TT * 2, dobytes = nvc * 64 * G * TT * 2;
            const uint32_t kbytes = nqc * 64 * kKV * 2, vbytes = do_dk ? nvc * 64 * kKV * 2 : 0;
            constexpr uint32_t id_s = idesc_f16(kBF16, 128, 64, false, false);
            const uint32_t id_v = idesc_f16(kBF16, 128, p.d2, false, true);
            const uint32_t id_k = idesc_f16(kBF16, 128, p.d1, false, true);
            bool ok = true;
            const int krow = it.cmp_row0 + it.kt * kKV;
            mbar_arrive_expect_tx(bar(B_KV0), kbytes + vbytes);
            for (int c = 0; c < nqc; ++c) tma_load_3d(ka + c * 16384, &tm_k, c * 64, it.group, krow, bar(B_KV0));
            if (do_dk)
                for (int c = 0; c < nvc; ++c) tma_load_3d(va + c * 16384, &tm_v, c * 64, it.group, krow, bar(B_KV0));
            // Q / dO M-tiles through a ring of p.nst stages.  A stage is refilled once the
            // dV/dK MMAs of the M-tile that last used it have retired (B_QE).
            auto load_q = [&](int mi) {
                const int st = mi % p.nst;
                const int row0 = it.q_row0 + mi * TT;
                const uint32_t qs0 = qa + st * p.stage_bytes, ds0 = doa + st * p.stage_bytes;
                mbar_arrive_expect_tx(bar(B_Q0 + st), qbytes + dobytes);
                for (int c = 0; c < nqc; ++c)
                    tma_load_3d(qs0 + c * 16384, &tm_q, c * 64, it.group * G, row0, bar(B_Q0 + st));
                for (int c = 0; c < nvc; ++c)
                    tma_load_3d(ds0 + c * 16384, &tm_do, c * 64, it.group * G, row0, bar(B_Q0 + st));
            };
            int loaded = 0;   // M-tiles whose loads have been issued
            auto ensure_loaded = [&](int m) {
                while (ok && loaded <= m && loaded < n_mt) {
                    const int st = loaded % p.nst;
                    if (loaded >= p.nst)
                        ok = mbar_wait(bar(B_QE0 + st), ((loaded / p.nst) - 1) & 1, sm.abort_flag, p.err,
                                       kErrTimeoutBase + 0x37);
                    if (!ok) break;
                    load_q(loaded++);
                }
            };
            ok = mbar_wait(bar(B_KV0), 0, sm.abort_flag, p.err, kErrTimeoutBase + 0x31);
            // Steps s = 2 mi + hf (halves of 64 query rows).  Step s uses score buffer
            // s % nsb (S^T at sb_col, dP^T at sb_col + 64).  With two buffers, S of step s + 1
            // is issued before the dV/dK of step s, so it runs while step s's softmax works;
            // the tensor core executes one thread's MMAs in issue order, so S of step s + 2
            // cannot overwrite P / dS of step s before its dV/dK has read them.
            const int nsb = p.nsb;
            auto sb_col = [&](int b) { return b == 0 ? 384u : 256u; };
            auto issue_s = [&](int step) {
                const int mi = step >> 1, hf = step & 1, st = mi % p.nst, b = step % nsb;
                if (hf == 0) {
                    ensure_loaded(mi);
                    ok = ok && mbar_wait(bar(B_Q0 + st), (mi / p.nst) & 1, sm.abort_flag, p.err,
                                         kErrTimeoutBase + 0x32);
                }
                if (!ok) return;
                const uint32_t qs = qa + st * p.stage_bytes, ds = doa + st * p.stage_bytes;
                tc_fence_after();
                for (int ks = 0; ks < p.d1 / 16; ++ks) {   // S^T = K Q^T over 64 query rows
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma_ss(tmem + sb_col(b), sdesc_sw128(ka + off, 16, 1024),
                            sdesc_sw128(qs + off + hf * 8192, 16, 1024), id_s, ks > 0 ? 1u : 0u);
                }
                if (do_dk)
                    for (int ks = 0; ks < p.d2 / 16; ++ks) {   // dP^T = V dO^T
                        const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                        umma_ss(tmem + sb_col(b) + 64, sdesc_sw128(va + off, 16, 1024),
                                sdesc_sw128(ds + off + hf * 8192, 16, 1024), id_s, ks > 0 ? 1u : 0u);
                    }
                umma_commit(bar(B_S0 + b));
            };
            auto issue_d = [&](int step) {
                const int mi = step >> 1, hf = step & 1, st = mi % p.nst, b = step % nsb;
                ok = ok && mbar_wait(bar(B_P0 + b), (step / nsb) & 1, sm.abort_flag, p.err, kErrTimeoutBase + 0x33);
                if (!ok) return;
                const uint32_t qs = qa + st * p.stage_bytes, ds = doa + st * p.stage_bytes;
                tc_fence_after();
                for (int ks = 0; ks < 64 / 16; ++ks) {
                    // the 64 query rows of the half are the contraction dimension: the
                    // row-major dO / Q chunks serve as MN-major operands
                    // Pᵀ / dSᵀ of query rows 32c .. 32c + 31 sit at the start of chunk c's
                    // columns (c = ks / 2), packed two to a column
                    const uint32_t pc = ks * 8 + (ks >= 2 ? 16 : 0);
                    if (do_dv)
                        umma_ts(tmem, tmem + sb_col(b) + pc, sdesc_sw128(ds + hf * 8192 + ks * 2048, 16384, 1024),
                                id_v, (step > 0 || ks > 0) ? 1u : 0u);
                    if (do_dk)
                        umma_ts(tmem + p.col_dk, tmem + sb_col(b) + 64 + pc,
                                sdesc_sw128(qs + hf * 8192 + ks * 2048, 16384, 1024), id_k,
                                (step > 0 || ks > 0) ? 1u : 0u);
                }
                if (hf == 1) umma_commit(bar(B_QE0 + st));
                // the next M-tile's load: its stage's last reader was issued a step ago
                if (p.nst == 2 && hf == 0) ensure_loaded(mi + 1);
            };
            const int total = 2 * n_mt;
            if (total > 0 && ok) issue_s(0);
            for (int step = 0; step < total && ok; ++step) {
                // S of the next step goes first when a second buffer holds it, except that with
                // one Q/dO stage the next M-tile's load waits for this step's dV/dK to retire
                const bool ahead = nsb == 2 && !(p.nst == 1 && ((step + 1) & 1) == 0);
                if (ahead && step + 1 < total) issue_s(step + 1);
                issue_d(step);
                if (!ahead && step + 1 < total) issue_s(step + 1);
            }
            // arrives once every MMA issued above has retired
            umma_commit(bar(B_DONE));
        }
    } else {
        // one key (compressed block) of the tile per thread; warps 0-3 take the first 32
        // query rows of each half-step, warps 5-8 the second, each in its lane quadrant
        const int quad = warp & 3, chalf = warp > 4 ? 1 : 0;
        const int kr = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int kb = it.kt * kKV + kr;   // block index inside the sequence
        const bool kvalid = kb < it.n_cmp;
        const float c2 = p.scale_log2;
        // this thread's row kr of M-tile mi: its statistics and visible count
        auto row_of = [&](int mi, float2& info, int& nv) {
            const int row0 = it.q_row0 + mi * TT;
            const int tok = kr / G, h = kr % G;
            const bool valid = kr < TT * G && row0 + tok < it.q_end;
            const int tpos = it.t0 + (row0 - it.q_row0) + tok;
            info = valid ? p.rowinfo[(size_t)(row0 + tok) * p.n1 + (size_t)it.group * G + h]
                         : make_float2(INFINITY, 0.f);
            nv = valid ? nvis_at(tpos, p.l, p.d, it.n_cmp) : 0;
        };
        if (n_mt > 0 && chalf == 0) row_of(0, rinfo2[kr], rnv2[kr]);
        for (int mi = 0; mi < n_mt; ++mi) {
            // buffer mi & 1 is complete, and M-tile mi - 1 (the other buffer) is no
            // longer read by anyone
            named_bar_sync(1, 256);
            const float2* rinfo = rinfo2 + (mi & 1) * 128;
            const int* rnv = rnv2 + (mi & 1) * 128;
            // the next M-tile's row, loaded now and stored after this M-tile's work
            float2 nxt_info = make_float2(INFINITY, 0.f);
            int nxt_nv = 0;
            if (mi + 1 < n_mt) row_of(mi + 1, nxt_info, nxt_nv);
            for (int hf = 0; hf < 2; ++hf) {
                const int step = mi * 2 + hf;
                const int b = step % p.nsb;
                const uint32_t scol = b == 0 ? 384u : 256u;   // S^T of this step's buffer, dP^T at + 64
                mbar_wait(bar(B_S0 + b), (step / p.nsb) & 1, sm.abort_flag, p.err, kErrTimeoutBase + 0x35);
                tc_fence_after();
                {
                    const int c = chalf;
                    uint32_t rs[32], rp[32];
                    tmem_ld32(tmem + lane_off + scol + c * 32, rs);
                    if (do_dk) tmem_ld32(tmem + lane_off + scol + 64 + c * 32, rp);
                    tmem_wait_ld_regs<32>(rs);
                    if (do_dk) tmem_wait_ld_regs<32>(rp);
                    uint32_t ppk[16], dpk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int r = hf * 64 + c * 32 + e;
                        const float2 i0 = rinfo[r], i1 = rinfo[r + 1];
                        const bool v0 = kvalid && kb < rnv[r], v1 = kvalid && kb < rnv[r + 1];
                        const float p0 = v0 ? ex2(__uint_as_float(rs[e]) * c2 - i0.x) : 0.f;
                        const float p1 = v1 ? ex2(__uint_as_float(rs[e + 1]) * c2 - i1.x) : 0.f;
                        ppk[e >> 1] = pk2<T>(p0, p1);
                        if (do_dk)
                            dpk[e >> 1] = pk2<T>(v0 ? p0 * (__uint_as_float(rp[e]) - i0.y) : 0.f,
                                                 v1 ? p1 * (__uint_as_float(rp[e + 1]) - i1.y) : 0.f);
                    }
                    // over this chunk's own Sᵀ / dPᵀ columns (the other warp reads the rest)
                    if (do_dv) tmem_st16(tmem + lane_off + scol + c * 32, ppk);
                    if (do_dk) tmem_st16(tmem + lane_off + scol + 64 + c * 32, dpk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_P0 + b));
            }
            if (mi + 1 < n_mt && chalf == 0) {
                rinfo2[((mi + 1) & 1) * 128 + kr] = nxt_info;
                rnv2[((mi + 1) & 1) * 128 + kr] = nxt_nv;
            }
        }
        mbar_wait(bar(B_DONE), 0, sm.abort_flag, p.err, kErrTimeoutBase + 0x36);
        tc_fence_after();
        // the run's partial sums; a run with no M-tile leaves zeros
        // (each of the quadrant's two warps stores half of the row's columns: dV then dK,
        // in 16-column pieces)
        float* dst = p.part + ((size_t)it.slot * 128 + kr) * (p.d1 + p.d2);
        const int ndv = do_dv ? p.d2 : 0, ndk = do_dk ? p.d1 : 0;
        const int np16 = (ndv + ndk) / 16, mine0 = chalf * ((np16 + 1) / 2) * 16,
                  mine1 = min(ndv + ndk, (chalf + 1) * ((np16 + 1) / 2) * 16);
        // column x of the row: dV for x < ndv, dK after (tensor memory: 0 and col_dk)
        auto seg = [&](int x0, int x1, bool zero) {
            if (x1 <= x0) return;
            const int xa = x0, xb = min(x1, ndv);
            if (xb > xa) {
                if (zero) {
                    for (int e = xa; e < xb; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(0.f, 0.f, 0.f, 0.f);
                } else {
                    store_row_f32(tmem + lane_off + xa, xb - xa, 1.f, dst + xa, true);
                }
            }
            const int ya = max(x0, ndv) - ndv, yb = x1 - ndv;
            if (yb > ya) {
                float* dk = dst + p.d2 + ya;
                if (zero) {
                    for (int e = 0; e < yb - ya; e += 4) *reinterpret_cast<float4*>(dk + e) = make_float4(0.f, 0.f, 0.f, 0.f);
                } else {
                    store_row_f32(tmem + lane_off + p.col_dk + ya, yb - ya, 1.f, dk, true);
                }
            }
        };
        if (!nsa_index_ok(it.slot < p.n_slots, p.err, 9)) {
        } else {
            seg(mine0, mine1, n_mt == 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*sm.abort_flag && threadIdx.x == 0) {
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 20000000ull) {
        }
    }
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dkcmp / dvcmp of one KV tile: its partial slots summed in slot order (a
// fixed order, so the result does not depend on the schedule); dK x scale.
__global__ void reduce_kernel(const KVTile* __restrict__ tiles, const float* __restrict__ part,
                              float* __restrict__ dkcmp, float* __restrict__ dvcmp, int n2, int d1, int d2,
                              float scale, long long rows_c, int* err) {
    const KVTile t = tiles[blockIdx.x];
    const int w = d1 + d2, w4 = w / 4;
    int rows = min(kKV, t.n_cmp - t.kt * kKV);
    if (!nsa_index_ok(t.cmp_row0 + t.kt * kKV + rows <= rows_c, err, 10)) rows = 0;
    for (int x = threadIdx.x; x < rows * w4; x += blockDim.x) {
        const int r = x / w4, c = (x % w4) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < t.nslots; ++s) {
            const float4 v = __ldcs(reinterpret_cast<const float4*>(part + ((size_t)(t.slot0 + s) * 128 + r) * w + c));
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        const size_t row = (size_t)(t.cmp_row0 + t.kt * kKV + r) * n2 + t.group;
        if (c < d2) {
            *reinterpret_cast<float4*>(dvcmp + row * d2 + c) = acc;
        } else {
            acc = make_float4(acc.x * scale, acc.y * scale, acc.z * scale, acc.w * scale);
            *reinterpret_cast<float4*>(dkcmp + row * d1 + (c - d2)) = acc;
        }
    }
}

cudaError_t launch_reduce(const KVTile* tiles, int ntiles, const float* part, float* dkcmp, float* dvcmp, int n2,
                          int d1, int d2, float scale, long long rows_c, int* err, cudaStream_t st) {
    if (ntiles <= 0) return cudaSuccess;
    reduce_kernel<<<ntiles, 256, 0, st>>>(tiles, part, dkcmp, dvcmp, n2, d1, d2, scale, rows_c, err);
    return cudaGetLastError();
}

template <typename K>
static cudaError_t launch_mma_kernel(K kern, const Params& p, int n, int threads, const CUtensorMap& tq,
                                     const CUtensorMap& tdo, const CUtensorMap& tk, const CUtensorMap& tv,
                                     cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
    if (e != cudaSuccess) return e;
    kern<<<n, threads, p.smem_bytes, st>>>(tq, tdo, tk, tv, p);
    return cudaGetLastError();
}

cudaError_t launch_dq(const Params& p, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                      const CUtensorMap& tv, cudaStream_t st) {
    return p.dtype == 0 ? launch_mma_kernel(dq_kernel<__nv_bfloat16>, p, p.n_qitems, kThreadsDq, tq, tdo, tk, tv, st)
                        : launch_mma_kernel(dq_kernel<__half>, p, p.n_qitems, kThreadsDq, tq, tdo, tk, tv, st);
}

cudaError_t launch_dkdv(const Params& p, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                        const CUtensorMap& tv, cudaStream_t st) {
    return p.dtype == 0 ? launch_mma_kernel(dkdv_kernel<__nv_bfloat16>, p, p.n_kvitems, kThreadsDq, tq, tdo, tk, tv, st)
                        : launch_mma_kernel(dkdv_kernel<__half>, p, p.n_kvitems, kThreadsDq, tq, tdo, tk, tv, st);
}

// ---------------------------------------------------- compression transposed

// dk[p] = sum_i w[p - i d] dkcmp_i over the windows i covering raw row p
// (dv likewise).  A CTA takes kRowsPerCta raw rows of one sequence; a thread
// one (head, 4 consecutive dims) column.  Walking its rows, a thread keeps
// the dkcmp values of the windows that cover the current row in registers
// (slot k: window q - k, q the row's group of d rows, position j = k d +
// row mod d in it) and loads one new window per group of d rows.
template <typename T, int BMAX>
__global__ void compress_dx_kernel(const CompressBwdParams p) {
    int s = 0;
    while (s + 1 < p.nseq && (int)blockIdx.x >= p.seq[s].blk_end) ++s;
    const CompressBwdSeq q = p.seq[s];
    const int blk0 = s ? p.seq[s - 1].blk_end : 0;
    const int r0 = ((int)blockIdx.x - blk0) * kRowsPerCta;
    const bool is_v = blockIdx.y == 1;
    const int dim = is_v ? p.d2 : p.d1;
    const float* __restrict__ g = is_v ? p.dvcmp : p.dkcmp;
    float* __restrict__ dx = is_v ? p.dv : p.dk;
    const T* __restrict__ w = reinterpret_cast<const T*>(p.w);
    const int ncol = p.n2 * dim / 4;
    const int l = p.l, d = p.d;
    const int nb = (l + d - 1) / d;   // windows covering a row, at most
    const int rows = min(kRowsPerCta, q.raw_len - r0);
    auto g_of = [&](int i, int n, int e) {   // dkcmp of window i (0 outside the sequence's windows)
        return (i >= 0 && i < q.n_cmp)
                   ? __ldg(reinterpret_cast<const float4*>(g + ((size_t)(q.cmp_start + i) * p.n2 + n) * dim + e))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    for (int col = threadIdx.x; col < ncol; col += blockDim.x) {
        const int n = (col * 4) / dim, e = (col * 4) % dim;
        int qg = r0 / d, rin = r0 - qg * d;
        float4 gq[BMAX];
#pragma unroll
        for (int k = 0; k < BMAX; ++k) gq[k] = (k < nb) ? g_of(qg - k, n, e) : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int rr = 0; rr < rows; ++rr) {
            const int pr = r0 + rr;   // raw row inside the sequence
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int k = 0; k < BMAX; ++k) {
                const int j = k * d + rin;
                if (k < nb && j < l) {
                    const float wv = static_cast<float>(w[(size_t)j * p.n2 + n]);
                    acc.x = fmaf(wv, gq[k].x, acc.x);
                    acc.y = fmaf(wv, gq[k].y, acc.y);
                    acc.z = fmaf(wv, gq[k].z, acc.z);
                    acc.w = fmaf(wv, gq[k].w, acc.w);
                }
            }
            if (nsa_index_ok(q.raw_start + pr < p.t2, nullptr, 11))
                // written once: stream past L2
                __stcs(reinterpret_cast<float4*>(dx + ((size_t)(q.raw_start + pr) * p.n2 + n) * dim + e), acc);
            if (++rin == d) {
                // the next group: every window moves one slot up, window qg + 1 enters slot 0
                rin = 0;
                ++qg;
#pragma unroll
                for (int k = BMAX - 1; k >= 1; --k) gq[k] = gq[k - 1];
                gq[0] = g_of(qg, n, e);
            }
        }
    }
}

// dw[j, n] = sum_i (dkcmp_i . k[i d + j] + dvcmp_i . v[i d + j]) over every
// compressed row i, in two steps.  Partial sums: a CTA takes a run of
// consecutive compressed rows [i0, i1) (p.dw_run of them, across sequence
// boundaries: cmp_raw gives each row's first raw row) and heads [y hpc,
// (y+1) hpc).  Thread (h, t) walks the run's groups of d raw rows, reading
// row t of each group once and adding it to every window of the run that
// covers it (window g - k at position j = k d + t, in slot k), as the forward
// compress does with its window sums; group g < i1 is window g's first group,
// the groups past i1 - 1 continue the last window's rows.  Then dw = the
// partials summed over the runs in run order (deterministic).
template <typename T, int BMAX>
__global__ void compress_dw_part_kernel(const CompressBwdParams p) {
    const int d = p.d, l = p.l;
    const int hpc = blockDim.x / d;
    const int h = threadIdx.x / d, t = threadIdx.x - h * d;
    const int n = blockIdx.y * hpc + h;
    if (h >= hpc || n >= p.n2) return;
    const int nb = (l + d - 1) / d;
    const long long i0 = (long long)blockIdx.x * p.dw_run;
    const long long i1 = min(i0 + p.dw_run, p.tc);
    const T* __restrict__ kk = reinterpret_cast<const T*>(p.k);
    const T* __restrict__ vv = reinterpret_cast<const T*>(p.v);
    float acc[BMAX];
#pragma unroll
    for (int k = 0; k < BMAX; ++k) acc[k] = 0.f;
    const long long last = p.cmp_raw[i1 - 1];
    for (long long g = i0; g < i1 + nb - 1; ++g) {
        const long long base = g < i1 ? (long long)p.cmp_raw[g] : last + (g - i1 + 1) * d;
        // the run's windows that hold row base + t, and where
        bool any = false;
        bool valid[BMAX];
#pragma unroll
        for (int k = 0; k < BMAX; ++k) {
            const long long wdx = g - k;
            valid[k] = k < nb && k * d + t < l && wdx >= i0 && wdx < i1 &&
                       (long long)p.cmp_raw[wdx] + (long long)k * d == base;
            any = any || valid[k];
        }
        if (!any) continue;
        const long long r = base + t;
        if (!nsa_index_ok(r < p.t2, nullptr, 12)) continue;
        const T* xk = kk + ((size_t)r * p.n2 + n) * p.d1;
        for (int e = 0; e < p.d1; e += 8) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(xk + e));
            const float2 a0 = up2<T>(u.x), a1 = up2<T>(u.y), a2 = up2<T>(u.z), a3 = up2<T>(u.w);
#pragma unroll
            for (int k = 0; k < BMAX; ++k) {
                if (!valid[k]) continue;
                const float* gk = p.dkcmp + ((size_t)(g - k) * p.n2 + n) * p.d1 + e;
                const float4 g0 = __ldg(reinterpret_cast<const float4*>(gk));
                const float4 g1 = __ldg(reinterpret_cast<const float4*>(gk + 4));
                acc[k] = fmaf(g0.x, a0.x, acc[k]);
                acc[k] = fmaf(g0.y, a0.y, acc[k]);
                acc[k] = fmaf(g0.z, a1.x, acc[k]);
                acc[k] = fmaf(g0.w, a1.y, acc[k]);
                acc[k] = fmaf(g1.x, a2.x, acc[k]);
                acc[k] = fmaf(g1.y, a2.y, acc[k]);
                acc[k] = fmaf(g1.z, a3.x, acc[k]);
                acc[k] = fmaf(g1.w, a3.y, acc[k]);
            }
        }
        if (p.dvcmp != nullptr) {
            const T* xv = vv + ((size_t)r * p.n2 + n) * p.d2;
            for (int e = 0; e < p.d2; e += 8) {
                const uint4 u = __ldg(reinterpret_cast<const uint4*>(xv + e));
                const float2 a0 = up2<T>(u.x), a1 = up2<T>(u.y), a2 = up2<T>(u.z), a3 = up2<T>(u.w);
#pragma unroll
                for (int k = 0; k < BMAX; ++k) {
                    if (!valid[k]) continue;
                    const float* gv = p.dvcmp + ((size_t)(g - k) * p.n2 + n) * p.d2 + e;
                    const float4 g0 = __ldg(reinterpret_cast<const float4*>(gv));
                    const float4 g1 = __ldg(reinterpret_cast<const float4*>(gv + 4));
                    acc[k] = fmaf(g0.x, a0.x, acc[k]);
                    acc[k] = fmaf(g0.y, a0.y, acc[k]);
                    acc[k] = fmaf(g0.z, a1.x, acc[k]);
                    acc[k] = fmaf(g0.w, a1.y, acc[k]);
                    acc[k] = fmaf(g1.x, a2.x, acc[k]);
                    acc[k] = fmaf(g1.y, a2.y, acc[k]);
                    acc[k] = fmaf(g1.z, a3.x, acc[k]);
                    acc[k] = fmaf(g1.w, a3.y, acc[k]);
                }
            }
        }
    }
    // every position j = k d + t of the run's partial row is this thread's
#pragma unroll
    for (int k = 0; k < BMAX; ++k)
        if (k < nb && k * d + t < l) p.dw_part[((size_t)blockIdx.x * l + k * d + t) * p.n2 + n] = acc[k];
}

// one warp per (j, n) of dw: lane k sums runs k, k + 32, ... in order, then a
// fixed butterfly sums the lanes
__global__ void compress_dw_reduce_kernel(const CompressBwdParams p, int nruns) {
    const int x = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);   // (j, n) of dw
    const int lane = threadIdx.x & 31;
    if (x >= p.l * p.n2) return;
    float acc = 0.f;
    for (int u = lane; u < nruns; u += 32) acc += p.dw_part[(size_t)u * p.l * p.n2 + x];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) p.dw[x] = acc;
}

cudaError_t launch_compress_bwd_dx(const CompressBwdParams& p, int blocks, cudaStream_t st) {
    if (blocks <= 0) return cudaSuccess;
    dim3 grid(blocks, p.dvcmp ? 2 : 1);
    const int nb = (p.l + p.d - 1) / p.d;
    const bool bf = p.dtype == 0;
#define NSA_DX(BM)                                                                          \
    {                                                                                      \
        if (bf) compress_dx_kernel<__nv_bfloat16, BM><<<grid, 256, 0, st>>>(p);            \
        else compress_dx_kernel<__half, BM><<<grid, 256, 0, st>>>(p);                      \
        return cudaGetLastError();                                                         \
    }
    if (nb <= 1) NSA_DX(1)
    if (nb <= 2) NSA_DX(2)
    if (nb <= 4) NSA_DX(4)
    NSA_DX(8)
#undef NSA_DX
}

int compress_dw_heads_per_cta(int d, int n2) { return std::max(1, std::min(256 / d, n2)); }

cudaError_t launch_compress_bwd_dw(const CompressBwdParams& p, int nruns, cudaStream_t st) {
    const int hpc = compress_dw_heads_per_cta(p.d, p.n2);
    if (nruns > 0) {
        dim3 grid(nruns, (p.n2 + hpc - 1) / hpc);
        const int nb = (p.l + p.d - 1) / p.d;
        const bool bf = p.dtype == 0;
#define NSA_DW(BM)                                                                          \
    {                                                                                      \
        if (bf) compress_dw_part_kernel<__nv_bfloat16, BM><<<grid, hpc * p.d, 0, st>>>(p); \
        else compress_dw_part_kernel<__half, BM><<<grid, hpc * p.d, 0, st>>>(p);           \
    }
        if (nb <= 1) NSA_DW(1)
        else if (nb <= 2) NSA_DW(2)
        else if (nb <= 4) NSA_DW(4)
        else NSA_DW(8)
#undef NSA_DW
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    compress_dw_reduce_kernel<<<(p.l * p.n2 + 7) / 8, 256, 0, st>>>(p, nruns);
    return cudaGetLastError();
}

}  // namespace bwd
}  // namespace nsa
