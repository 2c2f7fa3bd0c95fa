// art_order.cu -- importance-first traversal: page summaries, block scores and
// the walk order (art_page_summary, art_build_order_importance in art.h).
//
// "ART: Attention Run-time Termination for Efficient Large Language Model
// Decoding" (gist.science explainer), section 2.4: ART runs over a reordered
// traversal of the KV blocks, "recency-first" or "importance-first", with
// block 0 first.  The importance estimate is this library's own: the mean key
// of a page (one summary per page and kv-head, kept beside the cache) scored
// against the sum of the group's query heads.
//
// Three kernels, all HBM- or L2-bound gathers:
//   art_page_summary_kernel  one warp per (sequence, block, kv-head): streams
//                            the page's valid key rows with 16-byte loads and
//                            writes their mean.
//   art_block_score_kernel   one CTA per (sequence, run of blocks): the group
//                            sums of q sit in shared memory; each warp loads
//                            the page indices of its run at once and dots two
//                            blocks' summaries at a time with them.
//   art_rank_order_kernel    one CTA per (sequence, 64 blocks): each block's
//                            position is the number of blocks whose 64-bit
//                            (score, index) key sorts before its own, counted
//                            over all blocks of the sequence by 16 warps.  The
//                            keys are unique, so the order is a permutation
//                            for any scores and is bitwise reproducible.  It
//                            is launched as a programmatic dependent of the
//                            score kernel, so its launch overlaps that grid.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <type_traits>

#include "../../include/art.h"
#include "art_host.h"

namespace {

using art_host::aligned;
using art_host::elem_size;
using art_host::is_null;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRankChunk = 2048;   // keys staged in shared memory at a time (16 KiB)
constexpr int kRankThreads = 512;
constexpr int kRankWarps = kRankThreads / 32;
constexpr int kMaxQgFloats = 16384;

// ------------------------------------------------------ vector access ----

template <typename T>
struct Vec;

template <>
struct Vec<float> {
    static constexpr int E = 4;
    __device__ static __forceinline__ void load(const float *p, float *f)
    {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
        f[0] = v.x;
        f[1] = v.y;
        f[2] = v.z;
        f[3] = v.w;
    }
    __device__ static __forceinline__ void store(float *p, const float *f)
    {
        *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
    }
    __device__ static __forceinline__ float scalar(const float *p) { return __ldg(p); }
};

template <>
struct Vec<__nv_bfloat16> {
    static constexpr int E = 8;
    __device__ static __forceinline__ void load(const __nv_bfloat16 *p, float *f)
    {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static __forceinline__ void store(__nv_bfloat16 *p, const float *f)
    {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    __device__ static __forceinline__ float scalar(const __nv_bfloat16 *p)
    {
        return __bfloat162float(p[0]);
    }
};

// Writes VE means (VE = 4 or 8 consecutive channels) as TS.
template <typename TS, int VE>
__device__ __forceinline__ void store_mean(TS *dst, const float *m)
{
    if constexpr (std::is_same<TS, float>::value) {
#pragma unroll
        for (int s = 0; s < VE; s += 4)
            Vec<float>::store(dst + s, m + s);
    } else if constexpr (VE == 8) {
        Vec<__nv_bfloat16>::store(dst, m);
    } else {
        const __nv_bfloat162 h0 = __floats2bfloat162_rn(m[0], m[1]);
        const __nv_bfloat162 h1 = __floats2bfloat162_rn(m[2], m[3]);
        *reinterpret_cast<uint2 *>(dst) =
            make_uint2(*reinterpret_cast<const uint32_t *>(&h0), *reinterpret_cast<const uint32_t *>(&h1));
    }
}

__device__ __forceinline__ void report(int32_t *status, int32_t code)
{
    if (status)
        atomicCAS(status, 0, code);
}

// blocks of a sequence of L tokens, without the overflow of (L + page - 1)
// near INT32_MAX
__device__ __forceinline__ int n_blocks_of(int L, int page) { return L <= 0 ? 0 : L / page + (L % page != 0); }

// ------------------------------------------------------------ summary ----

struct SummaryArgs {
    const void *k;
    int64_t ks0, ks1, ks2;      // page, head, token strides (elements)
    const int32_t *pt;
    int64_t pts0;
    const int32_t *sl;
    void *sum;
    int64_t ss0, ss1;           // page, head strides (elements)
    int B, max_blocks, Hkv, page, d, num_pages;
    int32_t *status;
};

template <typename T, typename TS>
__global__ void __launch_bounds__(kThreads) art_page_summary_kernel(SummaryArgs a)
{
    constexpr int VE = Vec<T>::E;
    const int lane = threadIdx.x & 31;
    const int VR = a.d / VE;                          // 16-byte vectors per key row
    const int rpi = VR >= 32 ? 1 : 32 / VR;           // rows per warp iteration
    const int cpl = VR > 32 ? VR / 32 : 1;            // vectors per lane per row (<= 2)
    const int r0 = VR >= 32 ? 0 : lane / VR;
    const int cv0 = VR >= 32 ? lane : lane % VR;
    const int64_t items = (int64_t)a.B * a.max_blocks * a.Hkv;
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    for (int64_t it = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); it < items; it += nwarps) {
        const int h = (int)(it % a.Hkv);
        const int64_t bj = it / a.Hkv;
        const int j = (int)(bj % a.max_blocks);
        const int b = (int)(bj / a.max_blocks);
        const int L = a.sl[b];
        const int N = n_blocks_of(L, a.page);
        if (j == 0 && h == 0 && N > a.max_blocks)
            report(a.status, ART_ERR_BAD_INDEX);
        if (j >= N)
            continue;
        const int p = a.pt[(int64_t)b * a.pts0 + j];
        if (p < 0 || p >= a.num_pages) {
            if (h == 0)
                report(a.status, ART_ERR_BAD_INDEX);
            continue;
        }
        const int n = min(a.page, L - j * a.page);
        const T *base = static_cast<const T *>(a.k) + (int64_t)p * a.ks0 + (int64_t)h * a.ks1;
        float acc[2][VE];
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < VE; ++e)
                acc[c][e] = 0.f;
#pragma unroll 4
        for (int t = r0; t < n; t += rpi) {
            const T *row = base + (int64_t)t * a.ks2;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (c < cpl) {
                    float f[VE];
                    Vec<T>::load(row + (cv0 + 32 * c) * VE, f);
#pragma unroll
                    for (int e = 0; e < VE; ++e)
                        acc[c][e] += f[e];
                }
            }
        }
        // lanes that share a column vector hold partial sums of different rows
        for (int o = VR; o < 32; o <<= 1)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int e = 0; e < VE; ++e)
                    acc[c][e] += __shfl_xor_sync(0xffffffffu, acc[c][e], o);
        if (r0 == 0) {
            TS *dst = static_cast<TS *>(a.sum) + (int64_t)p * a.ss0 + (int64_t)h * a.ss1;
            const float fn = (float)n;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (c < cpl) {
                    float m[VE];
#pragma unroll
                    for (int e = 0; e < VE; ++e)
                        m[e] = acc[c][e] / fn;
                    store_mean<TS, VE>(dst + (cv0 + 32 * c) * VE, m);
                }
            }
        }
    }
}

// -------------------------------------------------------------- score ----

struct ScoreArgs {
    const void *q;
    int64_t qs0, qs1;
    const void *sum;
    int64_t ss0, ss1;
    const int32_t *pt;
    int64_t pts0;
    const int32_t *sl;
    float *scores;
    int64_t scs0;
    int B, Hq, Hkv, G, d, page, max_blocks, num_pages, blocks_per_warp;
    int q_vec;                  // q rows may be read 4 channels at a time (aligned)
    float scale;
    int32_t *status;
};

// 16 raw bytes of a summary row (8 bf16 or 4 fp32 channels), unpacked at use
template <typename TS>
__device__ __forceinline__ uint4 raw16(const TS *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

template <typename TS>
__device__ __forceinline__ void unpack16(const uint4 &v, float *f)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    if constexpr (std::is_same<TS, float>::value) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            f[i] = __uint_as_float(w[i]);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
}

// The query rows' group sums for 4 consecutive channels of head h:
// sum over g < G of q[h G + g][c .. c + 3] (fp32, in head order).
template <typename TQ>
__device__ __forceinline__ void group_sum4(const TQ *qb, int64_t qs1, int h, int G, int c, bool vec, float (&s)[4])
{
#pragma unroll
    for (int e = 0; e < 4; ++e)
        s[e] = 0.f;
    for (int g0 = 0; g0 < G; g0 += 4) {
        // four rows' reads in flight before any is added
        float f[4][4];
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                f[gg][e] = 0.f;
            if (g0 + gg < G) {
                const TQ *row = qb + (int64_t)(h * G + g0 + gg) * qs1 + c;
                if (vec) {
                    if constexpr (std::is_same<TQ, float>::value) {
                        const float4 v = __ldg(reinterpret_cast<const float4 *>(row));
                        f[gg][0] = v.x; f[gg][1] = v.y; f[gg][2] = v.z; f[gg][3] = v.w;
                    } else {
                        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(row));
                        f[gg][0] = __uint_as_float(v.x << 16);
                        f[gg][1] = __uint_as_float(v.x & 0xffff0000u);
                        f[gg][2] = __uint_as_float(v.y << 16);
                        f[gg][3] = __uint_as_float(v.y & 0xffff0000u);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        f[gg][e] = Vec<TQ>::scalar(row + e);
                }
            }
        }
#pragma unroll
        for (int gg = 0; gg < 4; ++gg)
            if (g0 + gg < G)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    s[e] += f[gg][e];
    }
}

// One warp scores NBW consecutive blocks of one sequence, two at a time
// (CH summary vectors of VE channels per lane and block).  The group sums of
// the query rows sit in shared memory, filled once per CTA; the page indices
// and the first pair's summaries are requested before that prologue, so its
// reads overlap theirs, and each later pair's summaries are requested while
// the previous pair is multiplied.  The arithmetic (group sums in head order,
// products vector by vector, a five-level butterfly) is fixed, so the scores
// are reproducible bit for bit.
template <typename TQ, typename TS, int CH>
__global__ void __launch_bounds__(kThreads, CH <= 2 ? 4 : 2) art_block_score_kernel(ScoreArgs a)
{
    extern __shared__ float qg[];   // [Hkv * d]: sum of the group's query heads
    constexpr int VE = Vec<TS>::E;
    // the rank kernel may launch now; its griddepcontrol.wait holds it until
    // this whole grid has finished and its stores are visible
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NBW = a.blocks_per_warp;                // even, at most 32
    const int jw = (blockIdx.x * kWarps + warp) * NBW;
    const int L = a.sl[b];
    int pidx = -1;
    if (lane < NBW && jw + lane < a.max_blocks)
        pidx = a.pt[(int64_t)b * a.pts0 + jw + lane];
    const int VR = a.d / VE;
    const int nv = a.Hkv * a.d / VE;                  // vectors per summary
    const int N = min(n_blocks_of(L, a.page), a.max_blocks);
    const TS *sb = static_cast<const TS *>(a.sum);
    // summaries of the pair starting at block jw + k (zeros where absent)
    auto fetch = [&](int k, uint4 (&ra)[CH], uint4 (&rb)[CH], bool &va, bool &vb) {
        const int ja = jw + k, jb = ja + 1;
        const int pa = __shfl_sync(0xffffffffu, pidx, k & 31);
        const int pbk = __shfl_sync(0xffffffffu, pidx, (k + 1) & 31);
        va = ja < N && pa >= 0 && pa < a.num_pages;
        vb = jb < N && pbk >= 0 && pbk < a.num_pages;
        const TS *ba = sb + (int64_t)(va ? pa : 0) * a.ss0;
        const TS *bbp = sb + (int64_t)(vb ? pbk : 0) * a.ss0;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int v = lane + 32 * c;
            const int h = v / VR, cv = v - h * VR;
            const int64_t off = (int64_t)h * a.ss1 + cv * VE;
            ra[c] = make_uint4(0u, 0u, 0u, 0u);
            rb[c] = make_uint4(0u, 0u, 0u, 0u);
            if (v < nv && va)
                ra[c] = raw16<TS>(ba + off);
            if (v < nv && vb)
                rb[c] = raw16<TS>(bbp + off);
        }
    };
    uint4 ca[CH], cb[CH];
    bool cva = false, cvb = false;
    if (jw < a.max_blocks)
        fetch(0, ca, cb, cva, cvb);   // in flight during the prologue below
    const int HD = a.Hkv * a.d;
    const TQ *qb = static_cast<const TQ *>(a.q) + (int64_t)b * a.qs0;
    for (int i4 = threadIdx.x; i4 < HD / 4; i4 += kThreads) {
        const int idx = i4 * 4, h = idx / a.d, c = idx - h * a.d;
        float sum4[4];
        group_sum4<TQ>(qb, a.qs1, h, a.G, c, a.q_vec != 0, sum4);
        *reinterpret_cast<float4 *>(qg + idx) = make_float4(sum4[0], sum4[1], sum4[2], sum4[3]);
    }
    __syncthreads();
    if (blockIdx.x == 0 && threadIdx.x == 0 && n_blocks_of(L, a.page) > a.max_blocks)
        report(a.status, ART_ERR_BAD_INDEX);
    if (jw >= a.max_blocks)
        return;                                       // no barrier follows
    float *srow = a.scores + (int64_t)b * a.scs0;
    for (int k = 0; k < NBW; k += 2) {
        const int ja = jw + k, jb = ja + 1;
        if (ja >= a.max_blocks)
            break;
        uint4 na[CH], nb2[CH];
        bool nva = false, nvb = false;
        if (k + 2 < NBW && ja + 2 < a.max_blocks)
            fetch(k + 2, na, nb2, nva, nvb);
        float acc_a = 0.f, acc_b = 0.f;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int v = lane + 32 * c;
            if (v < nv) {
                const int h = v / VR, cv = v - h * VR;
                const float *qv = qg + h * a.d + cv * VE;
                float fa[VE], fb[VE];
                unpack16<TS>(ca[c], fa);
                unpack16<TS>(cb[c], fb);
#pragma unroll
                for (int e = 0; e < VE; ++e) {
                    acc_a = fmaf(qv[e], fa[e], acc_a);
                    acc_b = fmaf(qv[e], fb[e], acc_b);
                }
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            acc_a += __shfl_xor_sync(0xffffffffu, acc_a, o);
            acc_b += __shfl_xor_sync(0xffffffffu, acc_b, o);
        }
        if (lane == 0) {
            const float nan = __int_as_float(0x7fc00000);
            float sa = ja >= N ? -INFINITY : (cva ? acc_a * a.scale : nan);
            if (sa == 0.f)
                sa = 0.f;   // -0 is stored as +0
            srow[ja] = sa;
            if ((ja < N && !cva) || (jb < N && !cvb))
                report(a.status, ART_ERR_BAD_INDEX);
            if (jb < a.max_blocks) {
                float sbv = jb >= N ? -INFINITY : (cvb ? acc_b * a.scale : nan);
                if (sbv == 0.f)
                    sbv = 0.f;
                srow[jb] = sbv;
            }
        }
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            ca[c] = na[c];
            cb[c] = nb2[c];
        }
        cva = nva;
        cvb = nvb;
    }
}

// Wide summaries (more than four vectors per lane): the group sums of the
// query rows sit in shared memory, filled by the whole CTA first.
template <typename TQ, typename TS, int CH>
__global__ void __launch_bounds__(kThreads, 2) art_block_score_wide_kernel(ScoreArgs a)
{
    // CH: summary vectors per lane and block kept in flight (1, 2 or 4)
    extern __shared__ float qg[];   // [Hkv * d]: sum of the group's query heads
    constexpr int VE = Vec<TS>::E;
    // the rank kernel may launch now; its griddepcontrol.wait holds it until
    // this whole grid has finished and its stores are visible
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NBW = a.blocks_per_warp;                // even, at most 32
    const int jw = (blockIdx.x * kWarps + warp) * NBW;
    // The sequence length, this warp's page indices (read up to the table's
    // width; entries past the sequence are ignored below) and the query rows
    // are independent reads: all of them go out before any is waited for.
    const int L = a.sl[b];
    int pidx = -1;
    if (lane < NBW && jw + lane < a.max_blocks)
        pidx = a.pt[(int64_t)b * a.pts0 + jw + lane];
    const int HD = a.Hkv * a.d;
    const TQ *qb = static_cast<const TQ *>(a.q) + (int64_t)b * a.qs0;
    for (int i4 = threadIdx.x; i4 < HD / 4; i4 += kThreads) {
        const int idx = i4 * 4, h = idx / a.d, c = idx - h * a.d;
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        for (int g0 = 0; g0 < a.G; g0 += 8) {         // up to 32 independent loads in flight
#pragma unroll
            for (int gg = 0; gg < 8; ++gg) {
                if (g0 + gg < a.G) {
                    const TQ *row = qb + (int64_t)(h * a.G + g0 + gg) * a.qs1 + c;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        s[e] += Vec<TQ>::scalar(row + e);
                }
            }
        }
        *reinterpret_cast<float4 *>(qg + idx) = make_float4(s[0], s[1], s[2], s[3]);
    }
    __syncthreads();
    const int N = min(n_blocks_of(L, a.page), a.max_blocks);
    if (jw + lane >= N)
        pidx = -1;
    if (blockIdx.x == 0 && threadIdx.x == 0 && n_blocks_of(L, a.page) > a.max_blocks)
        report(a.status, ART_ERR_BAD_INDEX);
    const int VR = a.d / VE;
    const int nv = HD / VE;                           // vectors per summary
    if (jw >= a.max_blocks)
        return;                                       // no barrier follows
    const TS *sb = static_cast<const TS *>(a.sum);
    float *srow = a.scores + (int64_t)b * a.scs0;
    for (int k = 0; k < NBW; k += 2) {                // two blocks at a time
        const int ja = jw + k, jb = ja + 1;
        if (ja >= a.max_blocks)
            break;
        const int pa = __shfl_sync(0xffffffffu, pidx, k);
        const int pb = __shfl_sync(0xffffffffu, pidx, k + 1);
        const bool va = ja < N && pa >= 0 && pa < a.num_pages;
        const bool vb = jb < N && pb >= 0 && pb < a.num_pages;
        const TS *ba = sb + (int64_t)(va ? pa : 0) * a.ss0;
        const TS *bb = sb + (int64_t)(vb ? pb : 0) * a.ss0;
        float acc_a = 0.f, acc_b = 0.f;
        for (int v0 = lane; v0 < nv; v0 += 32 * CH) {
            float fa[CH][VE], fb[CH][VE];
#pragma unroll
            for (int c = 0; c < CH; ++c) {
                const int v = v0 + 32 * c;
                const int h = v / VR, cv = v - h * VR;
                const int64_t off = (int64_t)h * a.ss1 + cv * VE;
#pragma unroll
                for (int e = 0; e < VE; ++e)
                    fa[c][e] = fb[c][e] = 0.f;
                if (v < nv && va)
                    Vec<TS>::load(ba + off, fa[c]);
                if (v < nv && vb)
                    Vec<TS>::load(bb + off, fb[c]);
            }
#pragma unroll
            for (int c = 0; c < CH; ++c) {
                const int v = v0 + 32 * c;
                if (v < nv) {
                    const int h = v / VR, cv = v - h * VR;
                    const float *qv = qg + h * a.d + cv * VE;
#pragma unroll
                    for (int e = 0; e < VE; ++e) {
                        acc_a = fmaf(qv[e], fa[c][e], acc_a);
                        acc_b = fmaf(qv[e], fb[c][e], acc_b);
                    }
                }
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            acc_a += __shfl_xor_sync(0xffffffffu, acc_a, o);
            acc_b += __shfl_xor_sync(0xffffffffu, acc_b, o);
        }
        if (lane == 0) {
            const float nan = __int_as_float(0x7fc00000);
            float sa = ja >= N ? -INFINITY : (va ? acc_a * a.scale : nan);
            if (sa == 0.f)
                sa = 0.f;   // -0 is stored as +0
            srow[ja] = sa;
            if ((ja < N && !va) || (jb < N && !vb))
                report(a.status, ART_ERR_BAD_INDEX);
            if (jb < a.max_blocks) {
                float sbv = jb >= N ? -INFINITY : (vb ? acc_b * a.scale : nan);
                if (sbv == 0.f)
                    sbv = 0.f;
                srow[jb] = sbv;
            }
        }
    }
}

// --------------------------------------------------------------- rank ----

struct RankArgs {
    const float *scores;
    int64_t scs0;
    const int32_t *sl;
    int page, max_blocks;
    int32_t *order;
    int64_t os0;
};

// Sorts ascending as: higher score first, equal scores larger index first.
// The float-to-integer map is monotone over all non-NaN values; -0 joins +0.
__device__ __forceinline__ unsigned long long order_key(float s, int j)
{
    uint32_t u = __float_as_uint(s);
    if ((u << 1) == 0u)
        u = 0u;
    const uint32_t mono = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)(~mono) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)j);
}

__global__ void __launch_bounds__(kRankThreads) art_rank_order_kernel(RankArgs a)
{
    // launched as a programmatic dependent of the score kernel: nothing it
    // reads may be touched before that grid has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ unsigned long long keys[kRankChunk];
    __shared__ int part[2][kRankWarps][32];
    const int b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int N = min(n_blocks_of(a.sl[b], a.page), a.max_blocks);
    const float *row = a.scores + (int64_t)b * a.scs0;
    // each lane ranks two blocks: i0 and i0 + 32
    const int i0 = blockIdx.x * 64 + lane, i1 = i0 + 32;
    const unsigned long long m0 = (i0 >= 1 && i0 < N) ? order_key(row[i0], i0) : ~0ull;
    const unsigned long long m1 = (i1 < N) ? order_key(row[i1], i1) : ~0ull;
    int c0n = 0, c1n = 0;
    if (blockIdx.x * 64 < N) {   // uniform over the CTA
        for (int c0 = 1; c0 < N; c0 += kRankChunk) {
            const int n = min(kRankChunk, N - c0);
            for (int t = threadIdx.x; t < n; t += kRankThreads)
                keys[t] = order_key(row[c0 + t], c0 + t);
            __syncthreads();
#pragma unroll 4
            for (int t = warp; t < n; t += kRankWarps) {
                const unsigned long long k = keys[t];
                c0n += k < m0 ? 1 : 0;
                c1n += k < m1 ? 1 : 0;
            }
            __syncthreads();
        }
    }
    part[0][warp][lane] = c0n;
    part[1][warp][lane] = c1n;
    __syncthreads();
    if (warp < 2) {
        const int i = warp == 0 ? i0 : i1;
        if (i < a.max_blocks) {
            int r = 0;
#pragma unroll
            for (int w = 0; w < kRankWarps; ++w)
                r += part[warp][w][lane];
            int32_t *out = a.order + (int64_t)b * a.os0;
            if (i >= N)
                out[i] = -1;
            else if (i == 0)
                out[0] = 0;
            else
                out[1 + r] = i;
        }
    }
}

// --------------------------------------------------------------- host ----

bool pow2_head_dim(int64_t d) { return d >= 16 && d <= 256 && (d & (d - 1)) == 0; }

bool float_type(int32_t dt) { return dt == ART_F32 || dt == ART_BF16; }

// 16-byte aligned base, positive strides that are multiples of 16 bytes, last dim contiguous
bool vec_layout(const art_tensor_t *t, int nd)
{
    const int64_t es = elem_size(t->dtype);
    if (!aligned(t->data, 16) || t->stride[nd - 1] != 1)
        return false;
    for (int i = 0; i < nd - 1; ++i)
        if (t->stride[i] <= 0 || (t->stride[i] * es) % 16)
            return false;
    return true;
}

art_status_t check_table(const art_tensor_t *pt, const art_tensor_t *sl, int64_t *B, int64_t *mb)
{
    if (pt->ndim != 2 || sl->ndim != 1)
        return ART_ERR_SHAPE;
    if (pt->dtype != ART_I32 || sl->dtype != ART_I32)
        return ART_ERR_DTYPE;
    *B = sl->shape[0];
    *mb = pt->shape[1];
    if (*B <= 0 || *B > 65535 || pt->shape[0] != *B || *mb <= 0 || *mb > (int64_t)INT32_MAX / 256 ||
        pt->stride[1] != 1 || pt->stride[0] < 0 || sl->stride[0] != 1)
        return ART_ERR_SHAPE;
    if (!aligned(pt->data, 4) || !aligned(sl->data, 4))
        return ART_ERR_SHAPE;
    return ART_OK;
}

int sm_count()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <typename T, typename TS>
void launch_summary(const SummaryArgs &a, int grid, cudaStream_t s)
{
    art_page_summary_kernel<T, TS><<<grid, kThreads, 0, s>>>(a);
}

template <typename TQ, typename TS, int CH>
cudaError_t launch_score_ch(const ScoreArgs &a, dim3 grid, size_t smem, cudaStream_t s)
{
    auto fn = art_block_score_kernel<TQ, TS, CH>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    fn<<<grid, kThreads, smem, s>>>(a);
    return cudaSuccess;
}

template <typename TQ, typename TS>
cudaError_t launch_score_wide(const ScoreArgs &a, dim3 grid, size_t smem, cudaStream_t s)
{
    auto fn = art_block_score_wide_kernel<TQ, TS, 4>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    fn<<<grid, kThreads, smem, s>>>(a);
    return cudaSuccess;
}

// loads in flight per lane and block: just enough to cover one summary
template <typename TQ, typename TS>
cudaError_t launch_score(const ScoreArgs &a, dim3 grid, size_t smem, cudaStream_t s)
{
    const int per_lane = (a.Hkv * a.d / Vec<TS>::E + 31) / 32;
    if (per_lane <= 1)
        return launch_score_ch<TQ, TS, 1>(a, grid, smem, s);
    if (per_lane == 2)
        return launch_score_ch<TQ, TS, 2>(a, grid, smem, s);
    if (per_lane <= 4)
        return launch_score_ch<TQ, TS, 4>(a, grid, smem, s);
    return launch_score_wide<TQ, TS>(a, grid, smem, s);
}

}  // namespace

extern "C" {

art_status_t art_page_summary(const art_tensor_t *k_cache, const art_tensor_t *page_table,
                              const art_tensor_t *seq_lens, art_tensor_t *summary, int32_t *device_status,
                              art_stream_t stream)
{
    if (is_null(k_cache) || is_null(page_table) || is_null(seq_lens) || is_null(summary))
        return ART_ERR_NULL;
    if (k_cache->ndim != 4 || summary->ndim != 3)
        return ART_ERR_SHAPE;
    if (!float_type(k_cache->dtype) || !float_type(summary->dtype))
        return ART_ERR_DTYPE;
    int64_t B, mb;
    const art_status_t st = check_table(page_table, seq_lens, &B, &mb);
    if (st != ART_OK)
        return st;
    const int64_t NP = k_cache->shape[0], Hkv = k_cache->shape[1], page = k_cache->shape[2], d = k_cache->shape[3];
    if (NP <= 0 || NP > (int64_t)INT32_MAX || Hkv <= 0 || Hkv > 4096 || page <= 0 || page > 4096)
        return ART_ERR_SHAPE;
    if (summary->shape[0] != NP || summary->shape[1] != Hkv || summary->shape[2] != d)
        return ART_ERR_SHAPE;
    if (!pow2_head_dim(d))
        return ART_ERR_UNSUPPORTED;
    if (!vec_layout(k_cache, 4) || !vec_layout(summary, 3) || (device_status && !aligned(device_status, 4)))
        return ART_ERR_SHAPE;
    SummaryArgs a;
    a.k = k_cache->data;
    a.ks0 = k_cache->stride[0];
    a.ks1 = k_cache->stride[1];
    a.ks2 = k_cache->stride[2];
    a.pt = static_cast<const int32_t *>(page_table->data);
    a.pts0 = page_table->stride[0];
    a.sl = static_cast<const int32_t *>(seq_lens->data);
    a.sum = summary->data;
    a.ss0 = summary->stride[0];
    a.ss1 = summary->stride[1];
    a.B = (int)B;
    a.max_blocks = (int)mb;
    a.Hkv = (int)Hkv;
    a.page = (int)page;
    a.d = (int)d;
    a.num_pages = (int)NP;
    a.status = device_status;
    const int64_t items = B * mb * Hkv;
    const int64_t want = (items + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)sm_count() * 8;
    const int grid = (int)(want < cap ? want : cap);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool kb = k_cache->dtype == ART_BF16, sb = summary->dtype == ART_BF16;
    if (kb && sb)
        launch_summary<__nv_bfloat16, __nv_bfloat16>(a, grid, s);
    else if (kb)
        launch_summary<__nv_bfloat16, float>(a, grid, s);
    else if (sb)
        launch_summary<float, __nv_bfloat16>(a, grid, s);
    else
        launch_summary<float, float>(a, grid, s);
    return cudaGetLastError() == cudaSuccess ? ART_OK : ART_ERR_LAUNCH;
}

art_status_t art_build_order_importance(const art_tensor_t *q, const art_tensor_t *summary,
                                        const art_tensor_t *page_table, const art_tensor_t *seq_lens, int32_t page,
                                        float sm_scale, art_tensor_t *block_scores, art_tensor_t *block_order,
                                        int32_t *device_status, art_stream_t stream)
{
    if (is_null(q) || is_null(summary) || is_null(page_table) || is_null(seq_lens) || is_null(block_scores) ||
        is_null(block_order))
        return ART_ERR_NULL;
    if (q->ndim != 3 || summary->ndim != 3 || block_scores->ndim != 2 || block_order->ndim != 2)
        return ART_ERR_SHAPE;
    if (!float_type(q->dtype) || !float_type(summary->dtype) || block_scores->dtype != ART_F32 ||
        block_order->dtype != ART_I32)
        return ART_ERR_DTYPE;
    int64_t B, mb;
    const art_status_t st = check_table(page_table, seq_lens, &B, &mb);
    if (st != ART_OK)
        return st;
    const int64_t Hq = q->shape[1], d = q->shape[2];
    const int64_t NP = summary->shape[0], Hkv = summary->shape[1];
    if (q->shape[0] != B || Hq <= 0 || Hkv <= 0 || NP <= 0 || NP > (int64_t)INT32_MAX || Hq % Hkv ||
        summary->shape[2] != d)
        return ART_ERR_SHAPE;
    if (block_scores->shape[0] != B || block_scores->shape[1] != mb || block_order->shape[0] != B ||
        block_order->shape[1] != mb || block_scores->stride[1] != 1 || block_order->stride[1] != 1 ||
        block_scores->stride[0] < 0 || block_order->stride[0] < 0)
        return ART_ERR_SHAPE;
    if (!aligned(block_scores->data, 4) || !aligned(block_order->data, 4) || (device_status && !aligned(device_status, 4)))
        return ART_ERR_SHAPE;
    if (q->stride[2] != 1 || q->stride[0] < 0 || q->stride[1] < 0 || !aligned(q->data, elem_size(q->dtype)) ||
        !vec_layout(summary, 3))
        return ART_ERR_SHAPE;
    if (page <= 0 || std::isnan(sm_scale) || std::isinf(sm_scale))
        return ART_ERR_PARAM;
    if (!pow2_head_dim(d) || Hkv * d > kMaxQgFloats)
        return ART_ERR_UNSUPPORTED;
    ScoreArgs a;
    a.q = q->data;
    a.qs0 = q->stride[0];
    a.qs1 = q->stride[1];
    a.sum = summary->data;
    a.ss0 = summary->stride[0];
    a.ss1 = summary->stride[1];
    a.pt = static_cast<const int32_t *>(page_table->data);
    a.pts0 = page_table->stride[0];
    a.sl = static_cast<const int32_t *>(seq_lens->data);
    a.scores = static_cast<float *>(block_scores->data);
    a.scs0 = block_scores->stride[0];
    a.B = (int)B;
    a.Hq = (int)Hq;
    a.Hkv = (int)Hkv;
    a.G = (int)(Hq / Hkv);
    a.d = (int)d;
    a.page = page;
    a.max_blocks = (int)mb;
    a.num_pages = (int)NP;
    a.scale = sm_scale > 0.f ? sm_scale : (float)(1.0 / std::sqrt((double)d));
    a.status = device_status;
    {
        // four channels per load where every q row starts on such a boundary
        const int64_t es = elem_size(q->dtype), vb = 4 * es;
        a.q_vec = aligned(q->data, (uintptr_t)vb) && (q->stride[0] * es) % vb == 0 && (q->stride[1] * es) % vb == 0;
    }
    // about four CTAs per SM over the whole batch; an even number of blocks per warp, at most 32
    const int64_t warps = (int64_t)sm_count() * 4 * kWarps;
    int64_t nbw = (B * mb + warps - 1) / warps;
    nbw = nbw < 2 ? 2 : (nbw > 32 ? 32 : nbw + (nbw & 1));
    a.blocks_per_warp = (int)nbw;
    const int64_t per = nbw * kWarps;
    const dim3 sgrid((unsigned)((mb + per - 1) / per), (unsigned)B);
    const size_t smem = (size_t)(Hkv * d) * sizeof(float);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool qb = q->dtype == ART_BF16, sb = summary->dtype == ART_BF16;
    cudaError_t e;
    if (qb && sb)
        e = launch_score<__nv_bfloat16, __nv_bfloat16>(a, sgrid, smem, s);
    else if (qb)
        e = launch_score<__nv_bfloat16, float>(a, sgrid, smem, s);
    else if (sb)
        e = launch_score<float, __nv_bfloat16>(a, sgrid, smem, s);
    else
        e = launch_score<float, float>(a, sgrid, smem, s);
    if (e != cudaSuccess || cudaGetLastError() != cudaSuccess)
        return ART_ERR_LAUNCH;
    RankArgs r;
    r.scores = a.scores;
    r.scs0 = a.scs0;
    r.sl = a.sl;
    r.page = page;
    r.max_blocks = (int)mb;
    r.order = static_cast<int32_t *>(block_order->data);
    r.os0 = block_order->stride[0];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((mb + 63) / 64), (unsigned)B);
    cfg.blockDim = dim3(kRankThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, art_rank_order_kernel, r) != cudaSuccess)
        return ART_ERR_LAUNCH;
    return cudaGetLastError() == cudaSuccess ? ART_OK : ART_ERR_LAUNCH;
}

}  // extern "C"
