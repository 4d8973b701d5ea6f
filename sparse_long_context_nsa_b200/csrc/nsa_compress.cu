// nsa_compress.cu -- sliding-window compression of raw K/V into block tokens.
//
// "aclnnNsaCompress", Formula section: block i of a sequence is
// phi(k[i*d .. i*d+l-1]) for 0 <= i <= floor((S-l)/d); phi is the weighted sum
// over the window with one weight per window position and head, the same
// weights for K and V.
//
// HBM-bound.  Each CTA owns a run of consecutive output blocks of one sequence
// and one tensor (K or V).  The raw rows of the run are contiguous in TND
// layout, so they are streamed through a shared-memory ring with 1D bulk
// copies (one copy moves a few rows of every head at once).  Every raw row is
// read from HBM once per CTA; the windows overlap in shared memory only, and the
// l - d rows two neighbouring runs share are read by both at about the same time
// (neighbours walk in opposite directions), the second read hitting L2.
// Each thread owns one 16-byte column vector (8 elements of one head) and
// keeps the partial sums of the <= ceil(l/d) windows that cover the current
// row in registers, shifting them by one slot at each group of d rows.
// fp32 accumulation in window order; one RNE rounding at the store.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "nsa_internal.h"
#include "ptx.cuh"

namespace nsa {

__device__ int g_compress_err = 0;

template <typename T>
__device__ __forceinline__ void cvt8(const uint4& u, float (&f)[8]);
template <>
__device__ __forceinline__ void cvt8<__nv_bfloat16>(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
template <>
__device__ __forceinline__ void cvt8<__half>(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
        float2 v = __half22float2(h);
        f[2 * i] = v.x;
        f[2 * i + 1] = v.y;
    }
}
template <typename T>
__device__ __forceinline__ uint4 pack8(const float (&f)[8]);
template <>
__device__ __forceinline__ uint4 pack8<__nv_bfloat16>(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}
template <>
__device__ __forceinline__ uint4 pack8<__half>(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <>
__device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }

// The stage loop of one run.  REV = false walks rows first to last, REV = true
// last to first.  In both directions the register slot k holds the window that
// started k groups of d rows before the current group q (window q - k), and the
// current row sits at position j = k d + (row mod d) inside it; walking forward a
// window is complete when its group of last rows is done, walking backward when
// its first row is.
template <typename T, int BMAX, bool REV>
__device__ __forceinline__ void compress_run(const CompressParams& p, const CompressSeq& sq, int i0, int i1,
                                             int nrows, int rowbytes, int rowelems, int dim,
                                             const char* gsrc, T* __restrict__ dst, const float* wsm,
                                             uint64_t* bars, volatile int* abort_flag, uint8_t* stages) {
    const int l = p.l, d = p.d;
    const int nb = (l + d - 1) / d;                  // windows covering one row
    const int nvec = rowelems / 8;                   // 16-byte vectors per row
    const int rs = p.rows_per_stage;
    const int nstage = (nrows + rs - 1) / rs;
    const int stage_bytes = rs * rowbytes;
    // stage n of the walk covers the run's stage REV ? nstage - 1 - n : n
    auto stage_of = [&](int n) { return REV ? nstage - 1 - n : n; };
    auto issue = [&](int n) {
        const int slot = n % kCompressStages;
        const int sg = stage_of(n);
        const int rows = min(rs, nrows - sg * rs);
        const uint32_t bytes = (uint32_t)(rows * rowbytes);
        const uint32_t bar = smem_u32(&bars[slot]);
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(smem_u32(stages + slot * stage_bytes), gsrc + (int64_t)sg * stage_bytes, bytes, bar);
    };
    if (threadIdx.x == 0) {
        for (int n = 0; n < kCompressStages && n < nstage; ++n) issue(n);
    }

    const int cv = threadIdx.x;                      // column vector of this thread
    const bool active = cv < nvec;
    const int head = active ? (cv * 8) / dim : 0;
    float acc[BMAX][8];
#pragma unroll
    for (int k = 0; k < BMAX; ++k)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;

    // the store of window i (the slot kk that holds it)
    auto store = [&](int i, int kk) {
        if (i < i0 || i >= i1) return;
        float o[8];
#pragma unroll
        for (int k = 0; k < BMAX; ++k)
            if (k == kk)
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = acc[k][e];
        int64_t orow = (int64_t)sq.cmp_start + i;
        bool ok_row = p.block_table != nullptr || nsa_index_ok(orow < p.tc_rows, &g_compress_err, 6);
        if (p.block_table != nullptr) {
            // the page comes from the caller's table: out-of-pool entries
            // are reported, never written through
            const int pg = p.block_table[(size_t)sq.seq * p.bt_stride + i / p.page_rows];
            ok_row = pg >= 0 && pg < p.num_pages;
            orow = (int64_t)pg * p.page_rows + i % p.page_rows;
            if (!ok_row) atomicCAS(&g_compress_err, 0, kErrBadPage);
        }
        if (ok_row) {
            T* out = dst + orow * rowelems + cv * 8;
            *reinterpret_cast<uint4*>(out) = pack8<T>(o);
        }
    };
    // one row at position j = k d + rin of window q - k, for every slot
    auto add_row = [&](const uint4& u, int rin) {
        float x[8];
        cvt8<T>(u, x);
#pragma unroll
        for (int k = 0; k < BMAX; ++k) {
            const int j = k * d + rin;
            if (k < nb && j < l) {
                const float wv = wsm[j * p.n2 + head];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[k][e] = fmaf(wv, x[e], acc[k][e]);
            }
        }
    };

    // forward: the group of the first row and the row's place in it; backward: the
    // same for the first of the last four rows (nrows, d and every stage's row
    // count are multiples of 4, so four rows never straddle a group)
    int q = REV ? i0 + (nrows - 4) / d : i0;
    int rin = REV ? (nrows - 4) % d : 0;
    int next_issue = min(kCompressStages, nstage);   // stages handed to the copy engine
    int n = 0;
    bool failed = false;
    for (; n < nstage; ++n) {
        const int slot = n % kCompressStages;
        const uint32_t parity = (uint32_t)((n / kCompressStages) & 1);
        const bool got = mbar_wait(smem_u32(&bars[slot]), parity, abort_flag, &g_compress_err,
                                   kErrTimeoutBase + 1);
        const int rows = min(rs, nrows - stage_of(n) * rs);
        const uint8_t* base = stages + slot * stage_bytes;
        if (active && got) {
            if constexpr (!REV) {
                // four rows per step: their loads are independent
                for (int r = 0; r < rows; r += 4) {
                    uint4 u[4];
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr)
                        u[rr] = *reinterpret_cast<const uint4*>(base + (r + rr) * rowbytes + cv * 16);
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) add_row(u[rr], rin + rr);
                    rin += 4;
                    const bool last_row = (n == nstage - 1) && (r + 4 == rows);
                    if (rin == d || last_row) {
                        // window q-(nb-1) has seen its last row: store it, shift slots up
                        store(q - (nb - 1), nb - 1);
#pragma unroll
                        for (int kk = BMAX - 1; kk >= 1; --kk)
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[kk][e] = acc[kk - 1][e];
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[0][e] = 0.f;
                        rin = 0;
                        ++q;
                    }
                }
            } else {
                for (int r = rows - 4; r >= 0; r -= 4) {
                    uint4 u[4];
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr)
                        u[rr] = *reinterpret_cast<const uint4*>(base + (r + rr) * rowbytes + cv * 16);
#pragma unroll
                    for (int rr = 3; rr >= 0; --rr) add_row(u[rr], rin + rr);
                    if (rin == 0) {
                        // window q has seen its first row: store it, shift slots down
                        store(q, 0);
#pragma unroll
                        for (int kk = 0; kk + 1 < BMAX; ++kk)
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[kk][e] = acc[kk + 1][e];
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[BMAX - 1][e] = 0.f;
                        rin = d - 4;
                        --q;
                    } else {
                        rin -= 4;
                    }
                }
            }
        }
        // every thread is done with this slot, and all agree whether the wait succeeded
        if (!__syncthreads_and(got ? 1 : 0)) { failed = true; break; }
        if (threadIdx.x == 0 && next_issue < nstage) issue(next_issue);
        if (next_issue < nstage) ++next_issue;
    }
    if (failed && threadIdx.x == 0) {
        // a wait gave up: let the copies still in flight land before the CTA exits
        for (int u = n; u < next_issue; ++u) {
            const uint32_t bar = smem_u32(&bars[u % kCompressStages]);
            const uint32_t parity = (uint32_t)((u / kCompressStages) & 1);
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < 100000000ull) {
            }
        }
    }
}

// One CTA = one run of output blocks [i0, i1) of one sequence of one tensor.
// BMAX >= ceil(l/d): number of register slots for overlapping windows.
template <typename T, int BMAX>
__global__ void __launch_bounds__(kCompressMaxThreads)
nsa_compress_kernel(const CompressParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    // --- locate the work item: blockIdx.y = tensor (0 = K, 1 = V) ---
    const int plane = blockIdx.y;
    const int dim = plane == 0 ? p.d1 : p.d2;
    const T* __restrict__ src = reinterpret_cast<const T*>(plane == 0 ? p.k : p.v);
    T* __restrict__ dst = reinterpret_cast<T*>(plane == 0 ? p.kcmp : p.vcmp);
    if (src == nullptr) return;
    int lo = 0, hi = p.nseq - 1;   // first sequence whose chunk prefix exceeds blockIdx.x
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (p.seq[mid].chunk_end > (int)blockIdx.x) hi = mid; else lo = mid + 1;
    }
    const CompressSeq sq = p.seq[lo];
    const int chunk = blockIdx.x - (sq.chunk_end - sq.nchunks);
    const int i0 = sq.first + chunk * p.chunk;
    const int i1 = min(i0 + p.chunk, sq.ncmp);
    if (i0 >= i1) return;

    const int l = p.l, d = p.d;
    const int rowelems = p.n2 * dim;
    const int rowbytes = rowelems * (int)sizeof(T);
    const int64_t rel0 = (int64_t)i0 * d;            // first raw row of the run (in seq)
    const int nrows = (i1 - 1 - i0) * d + l;         // raw rows of the run
    const char* gsrc = reinterpret_cast<const char*>(src) +
                       ((int64_t)sq.raw_start + rel0) * (int64_t)rowbytes;

    // --- shared memory: [weights fp32 l x n2][barriers][stages] ---
    float* wsm = reinterpret_cast<float*>(smem_raw);
    const int wbytes = ((l * p.n2 * 4) + 127) & ~127;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + wbytes);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem_raw + wbytes + 8 * kCompressStages);
    uint8_t* stages = smem_raw + wbytes + 128;

    const T* wsrc = reinterpret_cast<const T*>(p.w);
    for (int i = threadIdx.x; i < l * p.n2; i += blockDim.x) wsm[i] = to_f32<T>(wsrc[i]);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kCompressStages; ++s) mbar_init(smem_u32(&bars[s]), 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncthreads();

    // Adjacent runs walk their rows in opposite directions: a run and its neighbour
    // reach the l - d rows they share at about the same time (both at their ends, or
    // both at their starts), so the second read of those rows is an L2 hit instead of
    // a second trip to HBM.  (Up to four windows per row; with more, the backward
    // form's registers would spill, and every run walks forward.)
    if (BMAX <= 4 && (chunk & 1))
        compress_run<T, BMAX, true>(p, sq, i0, i1, nrows, rowbytes, rowelems, dim, gsrc, dst, wsm, bars,
                                     abort_flag, stages);
    else
        compress_run<T, BMAX, false>(p, sq, i0, i1, nrows, rowbytes, rowelems, dim, gsrc, dst, wsm, bars,
                                      abort_flag, stages);
}

template <typename T, int BMAX>
static cudaError_t launch_t(const CompressParams& p, dim3 grid, int threads, size_t smem,
                            cudaStream_t st) {
    auto kern = nsa_compress_kernel<T, BMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, threads, smem, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_compress(const CompressParams& p, dim3 grid, int threads, size_t smem,
                            cudaStream_t st) {
    const int nb = (p.l + p.d - 1) / p.d;
    const bool bf = p.dtype == 0;
#define NSA_DISPATCH(BM)                                                                     \
    return bf ? launch_t<__nv_bfloat16, BM>(p, grid, threads, smem, st)                      \
              : launch_t<__half, BM>(p, grid, threads, smem, st);
    if (nb <= 1) { NSA_DISPATCH(1) }
    if (nb <= 2) { NSA_DISPATCH(2) }
    if (nb <= 4) { NSA_DISPATCH(4) }
    NSA_DISPATCH(8)
#undef NSA_DISPATCH
}

cudaError_t read_compress_error(int* out, cudaStream_t st) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_compress_err, sizeof(int), 0, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess || *out == 0) return e;
    const int zero = 0;   // reported once: clear for the next call
    return cudaMemcpyToSymbol(g_compress_err, &zero, sizeof(int), 0, cudaMemcpyHostToDevice);
}

}  // namespace nsa
