// art_kernels.cuh -- ART run-time-terminated decode attention for sm_100a.
//
// Method: "ART: Attention Run-time Termination for Efficient Large Language
// Model Decoding" (gist.science explainer), Technical Summary section 2:
// 2.1 streaming tile-wise online-softmax accumulation, 2.2 the magnitude and
// direction statistics of the partial output and their thresholds, 2.3 the
// patience counter, 2.4 caller-chosen traversal order with the sink block
// always consumed.  The exact statistics are the relative magnitude change
// |‖o_j‖-‖o_{j-1}‖|/‖o_{j-1}‖ < eps_m and 1-cos(o_j,o_{j-1}) < eps_d over the
// concatenated outputs of the G query heads that share a kv head.
//
// Organisation (one cluster of C CTAs per (sequence, kv-head) unit):
//
//   producer warp   walks this CTA's share of the order (steps j = rank,
//                   rank+C, ...), fetches each page's K and V tiles with TMA
//                   into a ring of S stages, and never runs more than R steps
//                   ahead of the merged prefix (R = speculation window).  Once
//                   the stop is known it issues nothing more.
//   compute warps   turn one staged page into a block-local softmax state
//                   (m_j, l_j, u_j = P_j V_j / l_j per head), independent of all
//                   other blocks, and push it into the leader's ring slot j % R.
//   merge warp      (leader CTA only) folds the block states into the running
//                   output in walk order: o_j = o_{j-1} + beta_j (u_j - o_{j-1}),
//                   beta_j the block's share of the softmax mass.  The same pass
//                   forms the two statistics from Delta_j = o_j - o_{j-1} without
//                   cancellation, runs the patience rule and publishes the stop.
//
// Because every block state is exact on its own and the merge is sequential,
// the stop index is the one a strictly sequential walk would take; pages
// fetched past the stop are bounded by the window R.  Every wait is bounded by
// a timeout that raises an error flag instead of trapping.
#pragma once
#include <cuda_bf16.h>
#include <math_constants.h>

#include "art_ptx.cuh"

namespace art {

constexpr uint32_t kStopBit = 0x80000000u;
constexpr uint32_t kEndOfStream = 0xFFFFFFFFu;
constexpr int kMaxThreads = 352;  // producer + up to 4 merge + up to 6 compute warps
constexpr int kMaxComputeWarps = 6;
constexpr int kMinWindow = 8;     // at least one merge batch
constexpr int kRedFloats = 2 * 4 * 40;  // merge-warp exchange buffer
constexpr int kErrTimeout = -7;
constexpr int kErrBadIndex = -8;
constexpr int kEngineCuda = 1;
constexpr int kEngineMma = 2;

struct KernelArgs {
    const void *q;
    int64_t q_sb, q_sh;                 // element strides of q (d is contiguous)
    float *out;
    int64_t out_sb, out_sh;
    int32_t *stop_block;
    int64_t stop_sb, stop_sh;
    const int32_t *page_table;
    int64_t pt_sb;
    const int32_t *block_order;
    int64_t bo_sb;
    const int32_t *seq_lens;
    const float *eps_m_arr, *eps_d_arr;
    const int32_t *P_arr, *minb_arr;
    float eps_m, eps_d;
    int32_t P, min_blocks;
    float scale_log2;                   // softmax scale * log2(e)
    int32_t *blocks_fetched;
    int32_t *device_status;
    int32_t B, Hq, Hkv, G, num_pages, max_blocks;
    int32_t C, S, NW, R;                // cluster size, stages, compute warps, state-ring slots
    int32_t RF;                         // window: blocks fetched ahead of the merged prefix (>= R; above R
                                        // a finished block state waits for its slot)
    int32_t PF;                         // pages pulled into L2 ahead of the staged loads
    int64_t timeout_ns;
    int32_t debug_flags;
    // several query tokens per sequence sharing one walk (NQ = 1: one query);
    // G = NQ * GQ rows per unit, row r is head r % GQ of token r / GQ
    int32_t NQ, GQ;
    int64_t q_st, out_st, stop_st;      // element strides between a sequence's tokens
    // hand-over through a workspace in global memory (the walk whose merge
    // CTA is not in the fetching CTAs' cluster): per unit the merged count,
    // per fetching CTA its fetch count, per ring slot a ready tag and the
    // block state.  Every word carries this call's epoch in its high half.
    unsigned long long *g_ctrl, *g_done, *g_flags;
    float *g_states;
    uint32_t epoch;
    int32_t Rg, W;                      // global ring slots per unit, fetching CTAs per unit
};

// merged count of a unit published in the workspace during this call (0 before)
__device__ __forceinline__ uint32_t gm_merged(const KernelArgs &a, int unit)
{
    const unsigned long long v = ld_acquire_gpu_u64(a.g_ctrl + unit);
    return (uint32_t)(v >> 32) == a.epoch ? (uint32_t)v : 0u;
}

// Shared-memory carve-up, identical on host and device.
struct Layout {
    uint32_t tile_bytes, stage_bytes;
    uint32_t kv_off, ring_off, slot_bytes, u_off_floats;
    uint32_t pbuf_off, red_off, meta_off, bar_off, ctrl_off, total;
};

__host__ __device__ inline uint32_t round_up_u32(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Layout make_layout(int S, int NW, int R, int page, int d, int esize, int gmax,
                                              bool pbuf)
{
    Layout L;
    L.tile_bytes = (uint32_t)(page * d * esize);
    L.stage_bytes = 2 * L.tile_bytes;
    L.kv_off = 0;
    uint32_t off = S * L.stage_bytes;
    // slot: [flag, pad x3][m x gmax][l x gmax][pad][u x gmax*d]   (floats)
    L.u_off_floats = round_up_u32(4 + 2 * gmax, 4);
    L.slot_bytes = round_up_u32((L.u_off_floats + gmax * d) * 4, 16);
    L.ring_off = off;
    off += R * L.slot_bytes;
    L.pbuf_off = off;
    off += pbuf ? (uint32_t)(NW * page * gmax * 4) : 0u;
    L.red_off = off;
    off += kRedFloats * 4 + 16;  // merge-warp exchange: 2 batches x up to 4 warps x (32 sums, flag, norms),
                                 // then the batch size merge warp 0 chose, per batch parity
    L.meta_off = off;
    off += 2 * S * 4;  // stage_j[S], stage_nv[S]
    off = round_up_u32(off, 8);
    L.bar_off = off;
    off += (3 * S + R + 1) * 8;  // full_k, full_v, empty, ready, never
    L.ctrl_off = off;
    off += 16;  // ctrl, fetched, abort, pad
    L.total = off;
    return L;
}

__device__ __forceinline__ void record_error(int32_t *status, int code)
{
    if (status)
        atomicCAS(status, 0, code);
}

// Warp-wide bounded wait on an mbarrier phase.  Returns false (without
// trapping) when this CTA was told to abort or when timeout_ns passes; the
// latter also raises the abort flag and records the timeout.
template <bool kClusterAcquire>
__device__ __noinline__ bool warp_wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t *abort,
                                            int64_t timeout_ns, int32_t *status, bool respect_abort)
{
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        const bool ok = kClusterAcquire ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, ok))
            return true;
        if ((it & 7u) == 7u) {
            int quit = 0;
            if ((threadIdx.x & 31) == 0) {
                const uint64_t now = global_timer_ns();
                if (t0 == 0)
                    t0 = now;
                if (respect_abort && *abort) {
                    quit = 1;
                } else if ((int64_t)(now - t0) > timeout_ns) {
                    *abort = 1u;
                    record_error(status, kErrTimeout);
                    quit = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, quit, 0))
                return false;
        }
    }
}

template <bool kClusterAcquire>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile uint32_t *abort, int64_t timeout_ns,
                                          int32_t *status, bool respect_abort = true)
{
    const bool ok = kClusterAcquire ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ok))
        return true;
    return warp_wait_slow<kClusterAcquire>(bar, parity, abort, timeout_ns, status, respect_abort);
}

// ---- element loads ---------------------------------------------------------

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// DE consecutive elements of a shared-memory row starting at element lane*DE.
template <typename T, int DE>
__device__ __forceinline__ void load_chunk(const uint8_t *row, int lane, float (&f)[DE])
{
    if constexpr (sizeof(T) == 4) {
        const float *p = reinterpret_cast<const float *>(row) + lane * DE;
        if constexpr (DE == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(p);
            f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2 *>(p);
            f[0] = v.x; f[1] = v.y;
        }
    } else {
        const uint8_t *p = row + lane * DE * 2;
        if constexpr (DE == 4) {
            const uint2 v = *reinterpret_cast<const uint2 *>(p);
            f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
        } else {
            const uint32_t v = *reinterpret_cast<const uint32_t *>(p);
            f[0] = bf16_lo(v); f[1] = bf16_hi(v);
        }
    }
}

// Butterfly reduce-scatter of 32 per-lane partial sums: afterwards v[0] of
// lane l holds the warp-wide sum of entry l.
__device__ __forceinline__ void reduce_scatter32(float (&v)[32], int lane)
{
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
        const bool upper = (lane & k) != 0;
#pragma unroll
        for (int i = 0; i < k; ++i) {
            const float send = upper ? v[i] : v[i + k];
            const float keep = upper ? v[i + k] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
        }
    }
}

// Butterfly reduce-scatter of 16 per-lane partial sums: afterwards v[0] of
// lanes l and l+16 holds the warp-wide sum of entry l % 16.
__device__ __forceinline__ void reduce_scatter16(float (&v)[16], int lane)
{
#pragma unroll
    for (int k = 8; k >= 1; k >>= 1) {
        const bool upper = (lane & k) != 0;
#pragma unroll
        for (int i = 0; i < k; ++i) {
            const float send = upper ? v[i] : v[i + k];
            const float keep = upper ? v[i + k] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
        }
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 16);
}

// Byte offset of bf16 element (t, d) in a K or V tile stored as d/64 column
// slabs of [page][64] with the 128-byte TMA swizzle (16-byte chunk index
// XOR row mod 8).
template <int PAGE>
__device__ __forceinline__ uint32_t swz128(int t, int d)
{
    return (uint32_t)((d >> 6) * PAGE * 128 + t * 128 + ((((d & 63) >> 3) ^ (t & 7)) << 4) + (d & 7) * 2);
}

// ---- shared state handed to the roles ---------------------------------------

struct Shared {
    uint8_t *kv;          // S stages of [K tile | V tile]
    float *ring;          // R slots (meaningful in the leader)
    float *pbuf;          // per compute warp [PAGE][GMAX] (CUDA-core engine)
    float *red;           // merge-warp exchange
    uint32_t *stage_j, *stage_nv;
    // shared addresses of the mbarrier arrays
    uint32_t bar_full_k, bar_full_v, bar_empty, bar_ready, bar_never;
    // this CTA's shared addresses at which the leader (rank 0) keeps its state
    // ring and the ring's ready barriers (mapped to rank 0 with mapa)
    uint32_t ring_leader, ready_leader;
    volatile uint32_t *ctrl, *fetched, *abort;
    Layout L;
    __device__ uint32_t full_k(int s) const { return bar_full_k + 8u * s; }
    __device__ uint32_t full_v(int s) const { return bar_full_v + 8u * s; }
    __device__ uint32_t empty(int s) const { return bar_empty + 8u * s; }
    __device__ uint32_t ready(int r) const { return bar_ready + 8u * r; }
    __device__ uint32_t never() const { return bar_never; }
};

// ---- producer ----------------------------------------------------------------

// rank, C: this CTA's place among the CTAs that fetch for the unit and their
// number (steps j = rank, rank + C, ... are this CTA's).  CTRL: where the
// merged progress is read: 0 the cluster leader's shared memory (relaxed), 1
// the same with acquire semantics (needed where the warp that publishes it is
// not the one that read the freed slots), 2 the workspace in global memory.
template <typename T, int D, int PAGE, int ENGINE, int CTRL = 0>
__device__ void producer_role(const KernelArgs &a, const Shared &sh, const CUtensorMap *tmk, const CUtensorMap *tmv,
                              int b, int h, int N, int Lseq, uint32_t rank, int C, int first_lb, int first_pp)
{
    const int lane = threadIdx.x & 31;
    const int S = a.S, R = a.RF;
    const uint32_t ctrl_cl = mapa(smem_u32((const void *)sh.ctrl), 0);
    const int32_t *bo = a.block_order ? a.block_order + (int64_t)b * a.bo_sb : nullptr;
    const int32_t *pt = a.page_table + (int64_t)b * a.pt_sb;
    if (lane == 0) {
        prefetch_tensormap(tmk);
        prefetch_tensormap(tmv);
    }
    uint32_t issued = 0;        // stages handed out (pages, markers)
    uint32_t kphase = 0, vphase = 0;  // bit s: parity of the last phase armed on full_k[s] / full_v[s]
    uint32_t kused = 0, vused = 0;
    uint32_t touched = 0;        // this CTA's walk steps whose page was read (loaded or prefetched)
    // the first 32 index pairs were loaded before the set-up barriers
    int batch_k0 = 0, my_lb = first_lb, my_pp = first_pp;
    // L2 prefetch front: step k + PFS, PFS = ceil(PF / C) of this CTA's steps
    const int PFS = (a.PF + C - 1) / C;
    int pbatch_k0 = -1, my_plb = -1, my_ppp = -1;
    uint32_t ctrl_cache = 0;
    bool aborted = false;

    auto take_stage = [&](uint32_t i) -> bool {  // wait until stage i % S is free
        const int s = (int)(i % (uint32_t)S);
        if (i < (uint32_t)S)
            return true;
        return warp_wait<false>(sh.empty(s), ((i / S) - 1) & 1u, sh.abort, a.timeout_ns, a.device_status);
    };

    for (int k = 0;; ++k) {
        const int j = (int)rank + k * C;
        if (j >= N)
            break;
        if (batch_k0 < 0 || k - batch_k0 >= 32) {  // fetch the next 32 index pairs at once
            batch_k0 = k;
            const int jj = (int)rank + (k + lane) * C;
            my_lb = -1;
            my_pp = -1;
            if (jj < N) {
                // no order given: the sink block, then newest to oldest
                my_lb = a.block_order ? __ldg(bo + jj) : (jj == 0 ? 0 : N - jj);
                if (my_lb >= 0 && my_lb < N)
                    my_pp = __ldg(pt + my_lb);
            }
        }
        const int lb = __shfl_sync(0xffffffffu, my_lb, k - batch_k0);
        const int pp = __shfl_sync(0xffffffffu, my_pp, k - batch_k0);
        const bool bad = lb < 0 || lb >= N || pp < 0 || pp >= a.num_pages;

        // speculation window: step j only once j < merged + R.  The merged
        // count only grows, so a cached value is re-read when it no longer
        // admits j, and every fourth step to notice a stop early.
        int go = 1;
        if (lane == 0 && ((uint32_t)j >= ctrl_cache + (uint32_t)R || (k & 3) == 0)) {
            uint64_t t0 = 0;
            for (uint32_t it = 0;; ++it) {
                const uint32_t c = CTRL == 2   ? gm_merged(a, b * a.Hkv + h)
                                   : CTRL == 1 ? ld_acquire_cluster_u32(ctrl_cl)
                                               : ld_relaxed_cluster_u32(ctrl_cl);
                if (c & kStopBit) { go = 0; break; }
                ctrl_cache = c;
                if ((uint32_t)j < c + (uint32_t)R) break;
                if ((it & 15u) == 15u) {
                    const uint64_t now = global_timer_ns();
                    if (t0 == 0) t0 = now;
                    if (*sh.abort) { go = -1; break; }
                    if ((int64_t)(now - t0) > a.timeout_ns) {
                        *sh.abort = 1u;
                        record_error(a.device_status, kErrTimeout);
                        go = -1;
                        break;
                    }
                }
            }
        }
        go = __shfl_sync(0xffffffffu, go, 0);
        // every branch below that holds a warp collective must be warp-uniform:
        // give all lanes lane 0's view of the merged progress
        ctrl_cache = __shfl_sync(0xffffffffu, ctrl_cache, 0);
        if (go == 0)
            break;
        if (go < 0) { aborted = true; break; }
        if (!take_stage(issued)) { aborted = true; break; }
        const int s = (int)(issued % (uint32_t)S);
        if (lane == 0) {
            sh.stage_j[s] = (uint32_t)j;
            if (bad) {
                // pass the fault down the pipeline: the merge reports it
                sh.stage_nv[s] = 0xFFFFFFFFu;
                mbar_arrive(sh.full_k(s));
                mbar_arrive(sh.full_v(s));
                record_error(a.device_status, kErrBadIndex);
            } else {
                const int nv = min(PAGE, Lseq - lb * PAGE);
                sh.stage_nv[s] = (uint32_t)nv;
                const uint32_t kdst = smem_u32(sh.kv + (size_t)s * sh.L.stage_bytes);
                const uint32_t vdst = kdst + sh.L.tile_bytes;
                mbar_arrive_expect_tx(sh.full_k(s), sh.L.tile_bytes);
                if constexpr (ENGINE == kEngineMma) {
#pragma unroll
                    for (int sb = 0; sb < D / 64; ++sb)
                        tma_load_4d(kdst + sb * PAGE * 128, tmk, sb * 64, 0, h, pp, sh.full_k(s));
                } else {
                    tma_load_4d(kdst, tmk, 0, 0, h, pp, sh.full_k(s));
                }
                mbar_arrive_expect_tx(sh.full_v(s), sh.L.tile_bytes);
                if constexpr (ENGINE == kEngineMma) {
#pragma unroll
                    for (int sb = 0; sb < D / 64; ++sb)
                        tma_load_4d(vdst + sb * PAGE * 128, tmv, sb * 64, 0, h, pp, sh.full_v(s));
                } else {
                    tma_load_4d(vdst, tmv, 0, 0, h, pp, sh.full_v(s));
                }
            }
        }
        kphase ^= (kused >> s & 1u) ? (1u << s) : 0u;
        kused |= 1u << s;
        vphase ^= (vused >> s & 1u) ? (1u << s) : 0u;
        vused |= 1u << s;
        ++issued;
        if (bad)
            break;
        touched = max(touched, (uint32_t)k + 1u);
        // Keep the page PFS steps ahead warm in L2, within the window
        // extended by PF: pages read past the stop stay below R + PF.
        if (PFS > 0) {
            const int kp = k + PFS;
            const int jp = (int)rank + kp * C;
            if (jp < N && (uint32_t)jp < ctrl_cache + (uint32_t)(R + a.PF)) {
                if (pbatch_k0 < 0 || kp - pbatch_k0 >= 32) {
                    pbatch_k0 = kp;
                    const int jj = (int)rank + (kp + lane) * C;
                    my_plb = -1;
                    my_ppp = -1;
                    if (jj < N) {
                        my_plb = a.block_order ? __ldg(bo + jj) : (jj == 0 ? 0 : N - jj);
                        if (my_plb >= 0 && my_plb < N)
                            my_ppp = __ldg(pt + my_plb);
                    }
                }
                const int plb = __shfl_sync(0xffffffffu, my_plb, kp - pbatch_k0);
                const int ppp = __shfl_sync(0xffffffffu, my_ppp, kp - pbatch_k0);
                if (plb >= 0 && plb < N && ppp >= 0 && ppp < a.num_pages) {
                    if (lane == 0) {
                        if constexpr (ENGINE == kEngineMma) {
#pragma unroll
                            for (int sb = 0; sb < D / 64; ++sb) {
                                tma_prefetch_4d(tmk, sb * 64, 0, h, ppp);
                                tma_prefetch_4d(tmv, sb * 64, 0, h, ppp);
                            }
                        } else {
                            tma_prefetch_4d(tmk, 0, 0, h, ppp);
                            tma_prefetch_4d(tmv, 0, 0, h, ppp);
                        }
                    }
                    touched = max(touched, (uint32_t)kp + 1u);
                }
            }
        }
    }

    if (!aborted) {
        // one end-of-stream marker per compute warp, in issue order
        for (int w = 0; w < a.NW; ++w) {
            if (!take_stage(issued)) { aborted = true; break; }
            const int s = (int)(issued % (uint32_t)S);
            if (lane == 0) {
                sh.stage_j[s] = kEndOfStream;
                mbar_arrive(sh.full_k(s));
            }
            kphase ^= (kused >> s & 1u) ? (1u << s) : 0u;
            kused |= 1u << s;
            ++issued;
        }
    }
    if (aborted) {
        // let every copy already in flight land before shared memory goes away
        for (int s = 0; s < S; ++s) {
            if (kused >> s & 1u)
                warp_wait<false>(sh.full_k(s), kphase >> s & 1u, sh.abort, a.timeout_ns, a.device_status, false);
            if (vused >> s & 1u)
                warp_wait<false>(sh.full_v(s), vphase >> s & 1u, sh.abort, a.timeout_ns, a.device_status, false);
        }
    }
    if (lane == 0) {
        if constexpr (CTRL == 2)
            st_release_gpu_u64(a.g_done + (int64_t)(b * a.Hkv + h) * a.W + rank,
                               ((unsigned long long)a.epoch << 32) | touched);
        else
            atom_add_cluster_u32(mapa(smem_u32((const void *)sh.fetched), 0), touched);
    }
}

// ---- block engines -------------------------------------------------------------
//
// Each turns one staged page into (m_g, l_g, u_g) for the G query heads:
// m_g = max_t s_gt (log2 domain), l_g = sum_t 2^(s_gt - m_g),
// u_g = sum_t 2^(s_gt - m_g) v_t / l_g, and writes them to the leader's slot.

struct SlotRef {
    uint32_t base;   // cluster address of the slot
    uint32_t ready;  // cluster address of its ready barrier
    uint32_t need;   // the slot is free once the merged count reaches this (0: it is free)
    uint32_t ctrl;   // cluster address of the merged count
    // the same through the workspace: the slot, its ready tag and the tag
    // written there once the state is complete, the unit's merged count
    float *gslot;
    unsigned long long *gflag;
    unsigned long long tag;
    int unit;
};

// Wait (whole warp, bounded) until the slot a finished block state goes to
// is free: the block R places earlier in the walk has been merged.  Needed
// only where the window reaches past the state ring.  Takes and returns the
// last merged count this warp read (kStopBit set once the walk has stopped
// or failed: the state is then dropped), or kGateFailed on timeout or abort.
constexpr uint32_t kGateFailed = 0x7fffffffu;

static __device__ __noinline__ uint32_t slot_gate_wait(uint32_t need, uint32_t ctrl, uint32_t cache,
                                                       volatile uint32_t *abort, int64_t timeout_ns,
                                                       int32_t *status)
{
    if ((threadIdx.x & 31) == 0) {
        uint64_t t0 = 0;
        for (uint32_t it = 0;; ++it) {
            if ((cache & kStopBit) || cache >= need)
                break;
            cache = ld_acquire_cluster_u32(ctrl);
            if ((it & 15u) == 15u) {
                const uint64_t now = global_timer_ns();
                if (t0 == 0)
                    t0 = now;
                if (*abort) {
                    cache = kGateFailed;
                    break;
                }
                if ((int64_t)(now - t0) > timeout_ns) {
                    *abort = 1u;
                    record_error(status, kErrTimeout);
                    cache = kGateFailed;
                    break;
                }
            }
        }
    }
    cache = __shfl_sync(0xffffffffu, cache, 0);
    __syncwarp();  // the lanes' slot writes come after lane 0's acquire
    return cache;
}

// 1: push the state; 0: drop it (the walk has stopped); -1: timeout or abort
__device__ __forceinline__ int slot_gate(const KernelArgs &a, const Shared &sh, const SlotRef &sr, uint32_t &cache)
{
    cache = slot_gate_wait(sr.need, sr.ctrl, cache, sh.abort, a.timeout_ns, a.device_status);
    return cache == kGateFailed ? -1 : ((cache & kStopBit) ? 0 : 1);
}

// The same wait on the merged count in the workspace.
static __device__ __noinline__ uint32_t slot_gate_wait_gm(uint32_t need, const unsigned long long *ctrl,
                                                          uint32_t epoch, uint32_t cache, volatile uint32_t *abort,
                                                          int64_t timeout_ns, int32_t *status)
{
    if ((threadIdx.x & 31) == 0) {
        uint64_t t0 = 0;
        for (uint32_t it = 0;; ++it) {
            if ((cache & kStopBit) || cache >= need)
                break;
            const unsigned long long v = ld_acquire_gpu_u64(ctrl);
            cache = (uint32_t)(v >> 32) == epoch ? (uint32_t)v : 0u;
            if ((it & 15u) == 15u) {
                const uint64_t now = global_timer_ns();
                if (t0 == 0)
                    t0 = now;
                if (*abort) {
                    cache = kGateFailed;
                    break;
                }
                if ((int64_t)(now - t0) > timeout_ns) {
                    *abort = 1u;
                    record_error(status, kErrTimeout);
                    cache = kGateFailed;
                    break;
                }
            }
        }
    }
    return __shfl_sync(0xffffffffu, cache, 0);
}

__device__ __forceinline__ int slot_gate_gm(const KernelArgs &a, const Shared &sh, const SlotRef &sr, uint32_t &cache)
{
    cache = slot_gate_wait_gm(sr.need, a.g_ctrl + sr.unit, a.epoch, cache, sh.abort, a.timeout_ns, a.device_status);
    return cache == kGateFailed ? -1 : ((cache & kStopBit) ? 0 : 1);
}

// After the lanes' plain stores of a block state into the workspace: the
// state becomes visible before its ready tag (lane 0 orders the warp's stores
// it has synchronised with, then releases the tag).
__device__ __forceinline__ void gm_publish(const SlotRef &sr)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        __threadfence();
        st_release_gpu_u64(sr.gflag, sr.tag);
    }
}

// Bytes one block state occupies in a slot: flag word, m and l per head,
// and the normalised output u (all GMAX heads for the tensor-core layout,
// the G real heads for the CUDA-core layout).
__device__ __forceinline__ uint32_t slot_tx_bytes(int G, int D, int GMAX, int engine)
{
    return 4u + 8u * (uint32_t)G + 4u * (uint32_t)D * (uint32_t)(engine == kEngineMma ? GMAX : G);
}

// CUDA-core engine: lane l owns head-dim elements [l*DE, l*DE+DE).
template <typename T, int D, int PAGE, int GMAX>
struct CudaEngine {
    static constexpr int DE = D / 32;
    static constexpr int TB = 32 / GMAX;              // tokens per butterfly batch
    static constexpr int NB = (PAGE + TB - 1) / TB;   // batches per page
    float qf[GMAX][DE];

    __device__ void load_q(const KernelArgs &a, int b, int h, int lane)
    {
        const T *qp = reinterpret_cast<const T *>(a.q) + (int64_t)b * a.q_sb;
#pragma unroll
        for (int g = 0; g < GMAX; ++g)
#pragma unroll
            for (int e = 0; e < DE; ++e)
                qf[g][e] = (g < a.G) ? to_f32<T>(qp[(int64_t)(h * a.G + g) * a.q_sh + lane * DE + e]) : 0.f;
    }
    // several tokens per unit: row g is head g % GQ of token g / GQ
    __device__ void load_q_rows(const KernelArgs &a, int b, int h, int lane)
    {
        const T *qp = reinterpret_cast<const T *>(a.q) + (int64_t)b * a.q_sb;
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            const int t = g / a.GQ, gg = g - t * a.GQ;
            const T *row = qp + (int64_t)t * a.q_st + (int64_t)(h * a.GQ + gg) * a.q_sh;
#pragma unroll
            for (int e = 0; e < DE; ++e)
                qf[g][e] = (g < a.G) ? to_f32<T>(row[lane * DE + e]) : 0.f;
        }
    }

    // returns false on abort
    __device__ bool block(const KernelArgs &a, const Shared &sh, int s, uint32_t par, int nv, float *pbuf,
                          const SlotRef &sr, uint32_t u_off, int lane, uint32_t &gcache)
    {
        const uint8_t *kt = sh.kv + (size_t)s * sh.L.stage_bytes;
        const uint8_t *vt = kt + sh.L.tile_bytes;
        constexpr int ROWB = D * (int)sizeof(T);
        float sc[NB];
#pragma unroll
        for (int bt = 0; bt < NB; ++bt) {
            float v[32];
#pragma unroll
            for (int tt = 0; tt < TB; ++tt) {
                const int t = bt * TB + tt;
                if (t < PAGE) {
                    float kf[DE];
                    load_chunk<T, DE>(kt + t * ROWB, lane, kf);
#pragma unroll
                    for (int g = 0; g < GMAX; ++g) {
                        float acc = 0.f;
#pragma unroll
                        for (int e = 0; e < DE; ++e)
                            acc = fmaf(qf[g][e], kf[e], acc);
                        v[tt * GMAX + g] = acc;
                    }
                } else {
#pragma unroll
                    for (int g = 0; g < GMAX; ++g)
                        v[tt * GMAX + g] = 0.f;
                }
            }
            reduce_scatter32(v, lane);
            sc[bt] = v[0];
        }
        // lane holds the score of token bt*TB + lane/GMAX for head lane%GMAX
        const int gl = lane % GMAX;
        float m = -CUDART_INF_F;
#pragma unroll
        for (int bt = 0; bt < NB; ++bt) {
            const int t = bt * TB + lane / GMAX;
            const bool valid = (t < nv) && (gl < a.G);
            sc[bt] = valid ? sc[bt] * a.scale_log2 : -CUDART_INF_F;
            m = fmaxf(m, sc[bt]);
        }
#pragma unroll
        for (int off = 16; off >= GMAX; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float l = 0.f;
#pragma unroll
        for (int bt = 0; bt < NB; ++bt) {
            const int t = bt * TB + lane / GMAX;
            // ex2.approx: relative error below 2^-22, far inside the fp32 tolerance
            const float p = (sc[bt] == -CUDART_INF_F) ? 0.f : ex2_approx(sc[bt] - m);
            l += p;
            if (t < PAGE)
                pbuf[t * GMAX + gl] = p;
        }
#pragma unroll
        for (int off = 16; off >= GMAX; off >>= 1)
            l += __shfl_xor_sync(0xffffffffu, l, off);
        __syncwarp();

        if (!warp_wait<false>(sh.full_v(s), par, sh.abort, a.timeout_ns, a.device_status))
            return false;
        float acc[GMAX][DE];
#pragma unroll
        for (int g = 0; g < GMAX; ++g)
#pragma unroll
            for (int e = 0; e < DE; ++e)
                acc[g][e] = 0.f;
#pragma unroll 4
        for (int t = 0; t < nv; ++t) {
            float vf[DE];
            load_chunk<T, DE>(vt + t * ROWB, lane, vf);
            float pg[GMAX];
#pragma unroll
            for (int g = 0; g < GMAX; ++g)
                pg[g] = pbuf[t * GMAX + g];
#pragma unroll
            for (int g = 0; g < GMAX; ++g)
#pragma unroll
                for (int e = 0; e < DE; ++e)
                    acc[g][e] = fmaf(pg[g], vf[e], acc[g][e]);
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(sh.empty(s));

        // block state into the leader's slot, counted on its ready barrier
        if (sr.need) {
            const int g = slot_gate(a, sh, sr, gcache);
            if (g <= 0)
                return g == 0;
        }
        if (lane == 0) {
            mbar_arrive_expect_tx_cluster(sr.ready, slot_tx_bytes(a.G, D, GMAX, kEngineCuda));
            st_async_b32(sr.base, 0u, sr.ready);
        }
        if (lane < GMAX && lane < a.G) {
            st_async_b32(sr.base + 4u * (4 + lane), __float_as_uint(m), sr.ready);
            st_async_b32(sr.base + 4u * (4 + GMAX + lane), __float_as_uint(l), sr.ready);
        }
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            const float lg = __shfl_sync(0xffffffffu, l, g);
            if (g < a.G) {
                const float inv = lg > 0.f ? rcp_approx(lg) : 0.f;
                const uint32_t addr = sr.base + 4u * (u_off + g * D + lane * DE);
                if constexpr (DE == 4)
                    st_async_v4(addr, acc[g][0] * inv, acc[g][1] * inv, acc[g][2] * inv, acc[g][3] * inv,
                                sr.ready);
                else
                    st_async_v2(addr, acc[g][0] * inv, acc[g][1] * inv, sr.ready);
            }
        }
        return true;
    }
};

// Tensor-core engine (bf16): S^T = K q^T with mma.m16n8k16 (tokens x heads),
// then O^T = V^T P^T with P kept to ~16 significant bits as a bf16 hi + lo pair
// (for G <= 4 both halves share one n8 tile: columns 0-3 hi, 4-7 lo).
// SINK: 0 pushes block states into the cluster leader's shared memory, 1
// writes them into the workspace in global memory
template <int D, int PAGE, int GMAX, int SINK = 0>
struct MmaEngine {
    static constexpr int MT = PAGE / 16;  // token tiles
    static constexpr int KS = D / 16;     // head-dim tiles
    static constexpr bool kShared = GMAX <= 4;
    uint32_t qb[KS][2];

    __device__ void load_q(const KernelArgs &a, int b, int h, int lane)
    {
        const int r = lane >> 2, c = lane & 3;
        const __nv_bfloat16 *qp = reinterpret_cast<const __nv_bfloat16 *>(a.q) + (int64_t)b * a.q_sb;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qb[ks][0] = 0u;
            qb[ks][1] = 0u;
            if (r < a.G) {
                const __nv_bfloat16 *row = qp + (int64_t)(h * a.G + r) * a.q_sh + ks * 16 + 2 * c;
                qb[ks][0] = *reinterpret_cast<const uint32_t *>(row);
                qb[ks][1] = *reinterpret_cast<const uint32_t *>(row + 8);
            }
        }
    }
    // several tokens per unit: row r is head r % GQ of token r / GQ
    __device__ void load_q_rows(const KernelArgs &a, int b, int h, int lane)
    {
        const int r = lane >> 2, c = lane & 3;
        const int t = r / a.GQ, g = r - t * a.GQ;
        const __nv_bfloat16 *qp = reinterpret_cast<const __nv_bfloat16 *>(a.q) + (int64_t)b * a.q_sb +
                                  (int64_t)t * a.q_st + (int64_t)(h * a.GQ + g) * a.q_sh;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qb[ks][0] = 0u;
            qb[ks][1] = 0u;
            if (r < a.G) {
                const __nv_bfloat16 *row = qp + ks * 16 + 2 * c;
                qb[ks][0] = *reinterpret_cast<const uint32_t *>(row);
                qb[ks][1] = *reinterpret_cast<const uint32_t *>(row + 8);
            }
        }
    }

    __device__ bool block(const KernelArgs &a, const Shared &sh, int s, uint32_t par, int nv, float *,
                          const SlotRef &sr, uint32_t u_off, int lane, uint32_t &gcache)
    {
        const int r = lane >> 2, c = lane & 3;
        uint8_t *kt = sh.kv + (size_t)s * sh.L.stage_bytes;
        uint8_t *vt = kt + sh.L.tile_bytes;
        const uint32_t ku = smem_u32(kt), vu = smem_u32(vt);

        // scores, rows = tokens, columns = heads
        // (even and odd head-dim steps accumulate separately: shorter mma chains)
        // (head-dim steps outer, token tiles inner: 2*MT independent mma chains)
        float sacc[MT][4], sodd[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                sacc[mt][i] = sodd[mt][i] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks)
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int t = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int d = ks * 16 + (lane >> 4) * 8;
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(ku + swz128<PAGE>(t, d), a0, a1, a2, a3);
                mma_bf16_16816((ks & 1) ? sodd[mt] : sacc[mt], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
            }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                sacc[mt][i] += sodd[mt][i];
        // The max is taken on the raw scores (the scale is positive, so it
        // commutes with the max, bit for bit); each weight is then one fma and
        // one ex2.approx (relative error below 2^-22, far inside the ~16 bits
        // the bf16 hi + lo split of P keeps).
        const int g0 = 2 * c;
        const bool hv0 = g0 < a.G, hv1 = g0 + 1 < a.G;
        float m2[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = mt * 16 + r + (i >> 1) * 8;
                const bool valid = (t < nv) && ((i & 1) ? hv1 : hv0);
                sacc[mt][i] = valid ? sacc[mt][i] : -CUDART_INF_F;
                m2[i & 1] = fmaxf(m2[i & 1], sacc[mt][i]);
            }
#pragma unroll
        for (int off = 4; off <= 16; off <<= 1) {
            m2[0] = fmaxf(m2[0], __shfl_xor_sync(0xffffffffu, m2[0], off));
            m2[1] = fmaxf(m2[1], __shfl_xor_sync(0xffffffffu, m2[1], off));
        }
        m2[0] *= a.scale_log2;
        m2[1] *= a.scale_log2;
        float l2[2] = {0.f, 0.f};
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float sv = sacc[mt][i];
                const float p = (sv == -CUDART_INF_F) ? 0.f : ex2_approx(fmaf(sv, a.scale_log2, -m2[i & 1]));
                sacc[mt][i] = p;
                l2[i & 1] += p;
            }
#pragma unroll
        for (int off = 4; off <= 16; off <<= 1) {
            l2[0] += __shfl_xor_sync(0xffffffffu, l2[0], off);
            l2[1] += __shfl_xor_sync(0xffffffffu, l2[1], off);
        }

        // P as B operands: bh (hi, or hi|lo when shared), bl (lo, G > 4)
        uint32_t bh[MT][2], bl[MT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const float p0 = sacc[mt][2 * half], p1 = sacc[mt][2 * half + 1];
                const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
                const float2 hf = __bfloat1622float2(hi);
                const __nv_bfloat162 lo = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
                const uint32_t hu = *reinterpret_cast<const uint32_t *>(&hi);
                const uint32_t lu = *reinterpret_cast<const uint32_t *>(&lo);
                if constexpr (kShared) {
                    const uint32_t lo_from = __shfl_xor_sync(0xffffffffu, lu, 2);
                    bh[mt][half] = movmatrix_trans(c < 2 ? hu : lo_from);
                    bl[mt][half] = 0u;
                } else {
                    bh[mt][half] = movmatrix_trans(hu);
                    bl[mt][half] = movmatrix_trans(lu);
                }
            }

        if (!warp_wait<false>(sh.full_v(s), par, sh.abort, a.timeout_ns, a.device_status))
            return false;
        if (nv < PAGE) {
            // rows past the sequence end may hold anything: zero them so 0 * x = 0
            constexpr int CH = D / 64 * 8;  // 16-byte chunks per row
            for (int idx = lane; idx < (PAGE - nv) * CH; idx += 32) {
                const int t = nv + idx / CH, ch = idx % CH;
                *reinterpret_cast<uint4 *>(vt + (ch >> 3) * PAGE * 128 + t * 128 + (ch & 7) * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }
        // (token steps outer, head-dim tiles inner: KS independent mma chains)
        float oacc[KS][4], oacc2[KS][4];
#pragma unroll
        for (int dt = 0; dt < KS; ++dt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                oacc[dt][i] = oacc2[dt][i] = 0.f;
#pragma unroll
        for (int kt2 = 0; kt2 < MT; ++kt2)
#pragma unroll
            for (int dt = 0; dt < KS; ++dt) {
                const int t = kt2 * 16 + (lane & 7) + (lane >> 4) * 8;
                const int d = dt * 16 + ((lane >> 3) & 1) * 8;
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4_trans(vu + swz128<PAGE>(t, d), a0, a1, a2, a3);
                mma_bf16_16816(oacc[dt], a0, a1, a2, a3, bh[kt2][0], bh[kt2][1]);
                if constexpr (!kShared)
                    mma_bf16_16816(oacc2[dt], a0, a1, a2, a3, bl[kt2][0], bl[kt2][1]);
            }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(sh.empty(s));

        // columns of this lane after combining hi and lo: heads gA, gA+1
        const int gA = kShared ? 2 * (c & 1) : 2 * c;
        const bool writer = kShared ? (c < 2) : true;
        float tot[KS][4];
#pragma unroll
        for (int dt = 0; dt < KS; ++dt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if constexpr (kShared)
                    tot[dt][i] = oacc[dt][i] + __shfl_xor_sync(0xffffffffu, oacc[dt][i], 2);
                else
                    tot[dt][i] = oacc[dt][i] + oacc2[dt][i];
            }
        // slot layout of this engine: 16-byte vectors, vector (dt, r, c) holds
        // u[gA][d], u[gA+1][d], u[gA][d+8], u[gA+1][d+8] with d = 16 dt + r
        if (sr.need) {
            const int g = SINK ? slot_gate_gm(a, sh, sr, gcache) : slot_gate(a, sh, sr, gcache);
            if (g <= 0)
                return g == 0;
        }
        if constexpr (SINK == 1) {
            float *gs = sr.gslot;
            if (lane == 0)
                reinterpret_cast<uint32_t *>(gs)[0] = 0u;
            if (writer) {
                const bool w0 = gA < a.G, w1 = gA + 1 < a.G;
                const float inv0 = (w0 && l2[0] > 0.f) ? rcp_approx(l2[0]) : 0.f;
                const float inv1 = (w1 && l2[1] > 0.f) ? rcp_approx(l2[1]) : 0.f;
                if (r == 0) {
                    if (w0) {
                        gs[4 + gA] = m2[0];
                        gs[4 + GMAX + gA] = l2[0];
                    }
                    if (w1) {
                        gs[4 + gA + 1] = m2[1];
                        gs[4 + GMAX + gA + 1] = l2[1];
                    }
                }
                constexpr int WPT = kShared ? 16 : 32;
                const int widx = kShared ? (r * 2 + c) : (r * 4 + c);
#pragma unroll
                for (int dt = 0; dt < KS; ++dt)
                    *reinterpret_cast<float4 *>(gs + u_off + 4 * (dt * WPT + widx)) =
                        make_float4(tot[dt][0] * inv0, tot[dt][1] * inv1, tot[dt][2] * inv0, tot[dt][3] * inv1);
            }
            gm_publish(sr);
            return true;
        }
        if (lane == 0) {
            mbar_arrive_expect_tx_cluster(sr.ready, slot_tx_bytes(a.G, D, GMAX, kEngineMma));
            st_async_b32(sr.base, 0u, sr.ready);
        }
        if (writer) {
            const bool w0 = gA < a.G, w1 = gA + 1 < a.G;
            const float inv0 = (w0 && l2[0] > 0.f) ? rcp_approx(l2[0]) : 0.f;
            const float inv1 = (w1 && l2[1] > 0.f) ? rcp_approx(l2[1]) : 0.f;
            if (r == 0) {
                if (w0) {
                    st_async_b32(sr.base + 4u * (4 + gA), __float_as_uint(m2[0]), sr.ready);
                    st_async_b32(sr.base + 4u * (4 + GMAX + gA), __float_as_uint(l2[0]), sr.ready);
                }
                if (w1) {
                    st_async_b32(sr.base + 4u * (4 + gA + 1), __float_as_uint(m2[1]), sr.ready);
                    st_async_b32(sr.base + 4u * (4 + GMAX + gA + 1), __float_as_uint(l2[1]), sr.ready);
                }
            }
            constexpr int WPT = kShared ? 16 : 32;  // writer lanes per head-dim tile
            const int widx = kShared ? (r * 2 + c) : (r * 4 + c);
#pragma unroll
            for (int dt = 0; dt < KS; ++dt)
                st_async_v4(sr.base + 4u * (u_off + 4 * (dt * WPT + widx)), tot[dt][0] * inv0, tot[dt][1] * inv1,
                            tot[dt][2] * inv0, tot[dt][3] * inv1, sr.ready);
        }
        return true;
    }
};

template <typename T, int D, int PAGE, int GMAX, int ENGINE, int SINK = 0>
using EngineFor = typename std::conditional<ENGINE == kEngineMma, MmaEngine<D, PAGE, GMAX, SINK>,
                                            CudaEngine<T, D, PAGE, GMAX>>::type;

// eng holds the unit's queries, loaded before the set-up barriers.  GATE:
// the window reaches past the state ring, so a finished state waits for its
// slot (slot_gate).  SINK = 1: states go to the workspace ring (a.Rg slots
// per unit, always gated).
template <typename T, int D, int PAGE, int GMAX, int ENGINE, bool GATE = false, int SINK = 0>
__device__ void compute_role(const KernelArgs &a, const Shared &sh, int b, int h, int cw,
                             EngineFor<T, D, PAGE, GMAX, ENGINE, SINK> &eng)
{
    static_assert(SINK == 0 || ENGINE == kEngineMma, "the workspace sink is built for the tensor-core engine");
    const int lane = threadIdx.x & 31;
    float *pbuf = sh.pbuf + (ENGINE == kEngineMma ? 0 : cw * PAGE * GMAX);
    const uint32_t ring_cl = mapa(sh.ring_leader, 0);
    const uint32_t ready_cl = mapa(sh.ready_leader, 0);
    const uint32_t ctrl_cl = mapa(smem_u32((const void *)sh.ctrl), 0);
    uint32_t gcache = 0;
    for (uint32_t i = (uint32_t)cw;; i += (uint32_t)a.NW) {
        const int s = (int)(i % (uint32_t)a.S);
        const uint32_t par = (i / (uint32_t)a.S) & 1u;
        if (!warp_wait<false>(sh.full_k(s), par, sh.abort, a.timeout_ns, a.device_status))
            break;
        const uint32_t j = sh.stage_j[s];
        if (j == kEndOfStream)
            break;
        const int nv = (int)sh.stage_nv[s];
        SlotRef sr;
        if constexpr (SINK == 0) {
            const uint32_t slot = j % (uint32_t)a.R;
            sr.base = ring_cl + slot * sh.L.slot_bytes;
            sr.ready = ready_cl + 8u * slot;
            sr.need = (GATE && j >= (uint32_t)a.R) ? j - (uint32_t)a.R + 1u : 0u;
            sr.ctrl = ctrl_cl;
        } else {
            const int unit = b * a.Hkv + h;
            const uint32_t gslot = j % (uint32_t)a.Rg;
            sr.unit = unit;
            sr.gslot = a.g_states + ((int64_t)unit * a.Rg + gslot) * (sh.L.slot_bytes / 4);
            sr.gflag = a.g_flags + (int64_t)unit * a.Rg + gslot;
            sr.tag = ((unsigned long long)a.epoch << 32) | (unsigned long long)(j + 1u);
            sr.need = j >= (uint32_t)a.Rg ? j - (uint32_t)a.Rg + 1u : 0u;
        }
        if (nv < 0) {  // bad page: forward the flag, free the stage
            __syncwarp();
            if (lane == 0)
                mbar_arrive(sh.empty(s));
            if (sr.need) {
                const int g = SINK ? slot_gate_gm(a, sh, sr, gcache) : slot_gate(a, sh, sr, gcache);
                if (g < 0)
                    break;
                if (g == 0)
                    continue;
            }
            if constexpr (SINK == 1) {
                if (lane == 0)
                    reinterpret_cast<uint32_t *>(sr.gslot)[0] = 1u;
                gm_publish(sr);
            } else if (lane == 0) {
                mbar_arrive_expect_tx_cluster(sr.ready, 4u);
                st_async_b32(sr.base, 1u, sr.ready);
            }
            continue;
        }
        if (!eng.block(a, sh, s, par, nv, pbuf, sr, sh.L.u_off_floats, lane, gcache))
            break;
    }
}

// ---- merge -----------------------------------------------------------------------

// Which slot floats a merge lane owns.  The lane keeps the running output for
// NV vectors of VW floats; element e of vector i belongs to head
// head(lane, i, e) and head-dim index dim(lane, i, e).
template <int D, int GMAX, int ENGINE>
struct MergeLayout {  // CUDA-core slots: u[g][d]; lane owns d in [lane*DE, lane*DE+DE) of every head
    static constexpr int VW = D / 32, NV = GMAX;
    static constexpr bool kTwoHeads = false;
    __device__ static int off(int lane, int i) { return i * D + lane * VW; }
    __device__ static int head(int, int i, int) { return i; }
    __device__ static int dim(int lane, int, int e) { return lane * VW + e; }
};
template <int D, int GMAX>
struct MergeLayout<D, GMAX, kEngineMma> {  // tensor-core slots: vector v = dt*W + r*C + c
    static constexpr int W = GMAX <= 4 ? 16 : 32, CW = GMAX <= 4 ? 2 : 4;
    static constexpr int VW = 4, NV = (D / 16) * W / 32;
    static constexpr bool kTwoHeads = true;
    __device__ static int off(int lane, int i) { return 4 * (lane + 32 * i); }
    __device__ static int head(int lane, int, int e) { return 2 * (lane % CW) + (e & 1); }
    __device__ static int dim(int lane, int i, int e)
    {
        const int v = lane + 32 * i;
        return (v / W) * 16 + (v % W) / CW + (e >> 1) * 8;
    }
};

// How the merge is split: NM warps share the output elements (vectors
// [mw*NVW, mw*NVW+NVW) of every lane belong to merge warp mw); KB blocks are
// folded per batch; a scan lane holds one (block, head) pair, or two when
// eight heads fill a row of 32 lanes at four blocks.
template <int D, int GMAX, int ENGINE, int NMW>
struct MergeShape {
    using Lay = MergeLayout<D, GMAX, ENGINE>;
    // at least one warp per 16 floats of output a lane keeps (registers), at
    // most one per vector; all counts are powers of two
    static constexpr int TOT = Lay::NV * Lay::VW;
    static constexpr int NMIN = TOT / 16 < 1 ? 1 : TOT / 16;
    static constexpr int NM0 = NMW > NMIN ? NMW : NMIN;
    static constexpr int NM = NM0 < Lay::NV ? NM0 : Lay::NV;
    static constexpr int NVW = Lay::NV / NM;
    static constexpr int KB = 8;                  // blocks per merge batch
    static constexpr int KH = 32 / GMAX;          // blocks per row of scan lanes
    static constexpr int NH = KB > KH ? KB / KH : 1;  // (block, head) entries per scan lane
    static_assert(Lay::NV % NM == 0, "merge split");
    static_assert(NH * KH >= KB && NH <= 2, "scan rows");
};

__device__ __forceinline__ void merge_barrier(int nthreads)
{
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

__device__ __forceinline__ void merge_barrier2(int nthreads)
{
    asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory");
}

// Folds block states into the running output in walk order, KB blocks per
// batch.  Per batch: wait for the KB states; the scan lanes (one or two
// (block, head) pairs each) form the blocks' shares of the softmax mass with
// a prefix scan (block max, then prefix sums of l 2^(m - M)); every merge
// warp folds the blocks into its
// slice of o, accumulating ||o_{j-1}||^2, o_{j-1}.Delta_j and ||Delta_j||^2;
// the slices' sums meet in shared memory; every merge warp then evaluates the
// statistics of the batch's blocks lane-parallel and runs the patience rule,
// reaching the same decision.  A stop inside a batch replays the batch up to
// the stop from a snapshot, so the stop and the output are those of a
// strictly sequential walk.
//
// DET = false builds the same walk without the detector: the blocks are folded
// exactly as above (the same batches, shares and arithmetic, so the output
// equals the eps = 0 walk's bit for bit), but no statistic is formed, no
// patience rule runs and the walk never stops early.  It exists as the timing
// reference for the detector's cost.
template <int D, int GMAX, int ENGINE, int NMW, bool DET = true>
__device__ void merge_role(const KernelArgs &a, const Shared &sh, int b, int h, int N, int mw)
{
    using MS = MergeShape<D, GMAX, ENGINE, NMW>;
    using Lay = typename MS::Lay;
    constexpr int NVW = MS::NVW, VW = Lay::VW, KB = MS::KB, NM = MS::NM, KH = MS::KH, NH = MS::NH;
    static_assert(KB <= 8, "two partial sums per block in 16 lanes");
    const int lane = threadIdx.x & 31;
    const int G = a.G;
    const float eps_m = a.eps_m_arr ? a.eps_m_arr[b] : a.eps_m;
    const float eps_d = a.eps_d_arr ? a.eps_d_arr[b] : a.eps_d;
    const int P = a.P_arr ? a.P_arr[b] : a.P;
    const int minb = a.minb_arr ? a.minb_arr[b] : a.min_blocks;
    const uint32_t ctrl_cl = mapa(smem_u32((const void *)sh.ctrl), 0);
    const uint32_t u_off = sh.L.u_off_floats;
    const int slot_floats = (int)(sh.L.slot_bytes / 4);
    const int vbase = mw * NVW;

    // scan lane: blocks kl (and kl + KH) of the batch, head gl; it also keeps
    // the running softmax scalars of head gl
    const int kl = lane / GMAX, gl = lane % GMAX;
    float Mx = -CUDART_INF_F, Lm = 0.f;
    // running output of this lane's elements (element e of vector i).  Scalar
    // fp32: in these short dependent chains it runs faster than the packed
    // f32x2 forms, and rounds identically.
    float o[NVW][VW];
#pragma unroll
    for (int i = 0; i < NVW; ++i)
#pragma unroll
        for (int e = 0; e < VW; ++e)
            o[i][e] = 0.f;

    int cnt = 0, stop = 0;
    bool failed = false;
    if (a.debug_flags & 1) {
        // a wait nothing will ever satisfy: exercises the bounded-wait path
        if (!warp_wait<true>(sh.never(), 0u, sh.abort, a.timeout_ns, a.device_status))
            failed = true;
    }

    auto load_u = [&](const float *sp, float (&uv)[NVW][VW]) {
#pragma unroll
        for (int ii = 0; ii < NVW; ++ii) {
            const float *up = sp + u_off + Lay::off(lane, vbase + ii);
            if constexpr (VW == 4) {
                const float4 x = *reinterpret_cast<const float4 *>(up);
                uv[ii][0] = x.x;
                uv[ii][1] = x.y;
                uv[ii][2] = x.z;
                uv[ii][3] = x.w;
            } else {
                const float2 x = *reinterpret_cast<const float2 *>(up);
                uv[ii][0] = x.x;
                uv[ii][1] = x.y;
            }
        }
    };
    // Fold batch block k into this warp's slice: Delta = beta (u - o),
    // o += Delta; with sums, add o.Delta and |Delta|^2 of the slice to pd, pe
    // (accumulated over the even and the odd elements apart, then added).
    // b0, b1: the shares of the lane's two heads (two-head layouts).
    auto fold = [&](int k, float beta, float b0, float b1, const float (&uv)[NVW][VW], float &pd, float &pe,
                    bool sums) {
        float bp[NVW][2];
        const int kr = NH > 1 ? k % KH : k;  // row of the scan lanes holding block k
        if constexpr (Lay::kTwoHeads) {  // elements alternate between two heads
#pragma unroll
            for (int ii = 0; ii < NVW; ++ii) {
                bp[ii][0] = b0;
                bp[ii][1] = b1;
            }
        } else {  // vector i holds head i
#pragma unroll
            for (int ii = 0; ii < NVW; ++ii) {
                const float bi = __shfl_sync(0xffffffffu, beta, kr * GMAX + vbase + ii);
                bp[ii][0] = bp[ii][1] = (vbase + ii < G) ? bi : 0.f;
            }
        }
        float sd[2] = {0.f, 0.f}, se[2] = {0.f, 0.f};
#pragma unroll
        for (int ii = 0; ii < NVW; ++ii) {
            // the CUDA-core engine writes no state for padding rows (vector
            // i >= G): their slot floats are whatever the shared memory held,
            // so they are skipped, not weighted by 0 (0 * inf is NaN)
            if (!Lay::kTwoHeads && vbase + ii >= G)
                continue;
#pragma unroll
            for (int e = 0; e < VW; ++e) {
                // o += beta (u - o) as one fused step (one rounding), written
                // with explicit roundings so that every instantiation computes
                // exactly this
                const float bb = bp[ii][e & 1];
                const float df = __fsub_rn(uv[ii][e], o[ii][e]);
                if (sums) {
                    const float dl = __fmul_rn(bb, df);
                    sd[e & 1] = __fmaf_rn(o[ii][e], dl, sd[e & 1]);
                    se[e & 1] = __fmaf_rn(dl, dl, se[e & 1]);
                }
                o[ii][e] = __fmaf_rn(bb, df, o[ii][e]);
            }
        }
        if (sums) {
            pd = __fadd_rn(sd[0], sd[1]);
            pe = __fadd_rn(se[0], se[1]);
        }
    };
    // fold blocks 0..kend of the batch starting at slot s0 (u loads one block ahead)
    auto fold_batch = [&](int s0, int kend, float beta, float beta_hi, float (&v)[16], bool sums) {
        float ua[NVW][VW], ub[NVW][VW];
        load_u(sh.ring + (size_t)s0 * slot_floats, ua);
        // the shares of every block of the batch, fetched before the fold so
        // that the shuffles stay off the chain that carries o from block to block
        float bq0[KB], bq1[KB];
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            bq0[k] = bq1[k] = 0.f;
            if constexpr (Lay::kTwoHeads) {
                const float bk = (NH > 1 && k >= KH) ? beta_hi : beta;
                const int kr = NH > 1 ? k % KH : k;
                const int h0 = Lay::head(lane, 0, 0);
                bq0[k] = __shfl_sync(0xffffffffu, bk, kr * GMAX + h0);
                bq1[k] = __shfl_sync(0xffffffffu, bk, kr * GMAX + h0 + 1);
            }
        }
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            if (k > kend)
                break;
            if (k + 1 <= kend) {
                int sn = s0 + k + 1;
                sn = sn >= a.R ? sn - a.R : sn;
                load_u(sh.ring + (size_t)sn * slot_floats, (k & 1) ? ua : ub);
            }
            fold(k, (NH > 1 && k >= KH) ? beta_hi : beta, bq0[k], bq1[k], (k & 1) ? ub : ua, v[2 * k], v[2 * k + 1],
                 sums);
        }
    };

    int s0 = 0;        // slot of the batch's first block, j0 % R
    uint32_t ph0 = 0;  // parity of that slot's phase, (j0 / R) & 1
    for (int j0 = 0, batch = 0; !failed && stop == 0 && j0 < N; ++batch) {
        const int nmax = min(KB, N - j0);
        // 1. lane k polls block j0 + k until the whole batch has arrived.  A
        //    flagged state (bad order or page entry upstream) ends the walk at
        //    once: the blocks after it are never produced.
        int sk = s0 + (lane < KB ? lane : 0);
        uint32_t pk = ph0;
        if (sk >= a.R) {
            sk -= a.R;
            pk ^= 1u;
        }
        const float *spk = sh.ring + (size_t)sk * slot_floats;
        bool local_fail = false;
        int nb = 0;
        // Merge warp 0 alone polls; with several merge warps it hands the
        // batch size (or a failure) to the others, so that all of them fold
        // exactly the same blocks and meet at the same barriers.
        if (mw == 0) {
            uint64_t t0 = 0;
            for (uint32_t it = 0;; ++it) {
                const bool arrived = lane < nmax && mbar_try_wait(sh.ready(sk), pk);
                if (__any_sync(0xffffffffu, arrived && __float_as_uint(spk[0]) != 0u)) {
                    local_fail = true;
                    break;
                }
                // batches have fixed boundaries (multiples of KB), so the
                // arithmetic, and the result, never depend on arrival timing
                if (__all_sync(0xffffffffu, arrived || lane >= nmax)) {
                    nb = nmax;
                    break;
                }
                if ((it & 7u) == 7u) {
                    int quit = 0;
                    if (lane == 0) {
                        const uint64_t now = global_timer_ns();
                        if (t0 == 0)
                            t0 = now;
                        if (*sh.abort) {
                            quit = 1;
                        } else if ((int64_t)(now - t0) > a.timeout_ns) {
                            *sh.abort = 1u;
                            record_error(a.device_status, kErrTimeout);
                            quit = 1;
                        }
                    }
                    if (__shfl_sync(0xffffffffu, quit, 0)) {
                        local_fail = true;
                        break;
                    }
                }
            }
        }
        if constexpr (NM > 1) {
            volatile int *agreed = reinterpret_cast<volatile int *>(sh.red + 2 * 4 * 34) + (batch & 1);
            if (mw == 0 && lane == 0)
                *agreed = local_fail ? -1 : nb;
            merge_barrier2(NM * 32);
            const int v = *agreed;
            local_fail = v < 0;
            nb = v < 0 ? 0 : v;
        }
        float v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
            v[q] = 0.f;
        float beta = 0.f, beta_hi = 0.f, n0part = 0.f;  // beta_hi: blocks KH.. (two scan rows)
        float o0[NVW][VW];
        if (!local_fail) {
            // 2. shares of the softmax mass: beta_(k,g) = w_k / (L_prev + w_0 + ... + w_k)
            float Mb;
            if constexpr (NH == 1) {  // one (block, head) entry per lane
                float mk = -CUDART_INF_F, lk = 0.f;
                if (kl < nb && gl < G) {
                    int sl = s0 + kl;
                    sl = sl >= a.R ? sl - a.R : sl;
                    const float *sp = sh.ring + (size_t)sl * slot_floats;
                    mk = sp[4 + gl];
                    lk = sp[4 + GMAX + gl];
                }
                Mb = fmaxf(Mx, mk);
#pragma unroll
                for (int off = GMAX; off < 32; off <<= 1)
                    Mb = fmaxf(Mb, __shfl_xor_sync(0xffffffffu, Mb, off));
                // (explicitly rounded products: the compiler may not fuse them into a
                // later add, so every instantiation folds with the same arithmetic)
                const float w = (mk == -CUDART_INF_F) ? 0.f : __fmul_rn(lk, ex2_approx(mk - Mb));
                float S = w;
#pragma unroll
                for (int off = GMAX; off < 32; off <<= 1) {
                    const float t = __shfl_up_sync(0xffffffffu, S, off);
                    if (lane >= off)
                        S += t;
                }
                const float Lam = ((Mx == -CUDART_INF_F) ? 0.f : __fmul_rn(Lm, ex2_approx(Mx - Mb))) + S;
                beta = Lam > 0.f ? __fmul_rn(w, rcp_approx(Lam)) : 0.f;
                Lm = __shfl_sync(0xffffffffu, Lam, (nb - 1) * GMAX + gl);
            } else {  // two rows: entry hh of a lane is block kl + hh KH
                float mk[NH], lk[NH];
                Mb = Mx;
#pragma unroll
                for (int hh = 0; hh < NH; ++hh) {
                    const int k = kl + hh * KH;
                    mk[hh] = -CUDART_INF_F;
                    lk[hh] = 0.f;
                    if (k < nb && gl < G) {
                        int sl = s0 + k;
                        sl = sl >= a.R ? sl - a.R : sl;
                        const float *sp = sh.ring + (size_t)sl * slot_floats;
                        mk[hh] = sp[4 + gl];
                        lk[hh] = sp[4 + GMAX + gl];
                    }
                    Mb = fmaxf(Mb, mk[hh]);
                }
#pragma unroll
                for (int off = GMAX; off < 32; off <<= 1)
                    Mb = fmaxf(Mb, __shfl_xor_sync(0xffffffffu, Mb, off));
                float w[NH], S[NH];
#pragma unroll
                for (int hh = 0; hh < NH; ++hh) {
                    w[hh] = (mk[hh] == -CUDART_INF_F) ? 0.f : __fmul_rn(lk[hh], ex2_approx(mk[hh] - Mb));
                    S[hh] = w[hh];
                }
#pragma unroll
                for (int off = GMAX; off < 32; off <<= 1)
#pragma unroll
                    for (int hh = 0; hh < NH; ++hh) {
                        const float t = __shfl_up_sync(0xffffffffu, S[hh], off);
                        if (lane >= off)
                            S[hh] += t;
                    }
                if constexpr (NH > 1)  // the second row follows the whole first row
                    S[1] += __shfl_sync(0xffffffffu, S[0], (KH - 1) * GMAX + gl);
                const float base = (Mx == -CUDART_INF_F) ? 0.f : __fmul_rn(Lm, ex2_approx(Mx - Mb));
                float Lam[NH], bh[NH];
#pragma unroll
                for (int hh = 0; hh < NH; ++hh) {
                    Lam[hh] = base + S[hh];
                    bh[hh] = Lam[hh] > 0.f ? __fmul_rn(w[hh], rcp_approx(Lam[hh])) : 0.f;
                }
                beta = bh[0];
                beta_hi = bh[NH - 1];
                const float Llast = (NH > 1 && nb - 1 >= KH) ? Lam[NH - 1] : Lam[0];
                Lm = __shfl_sync(0xffffffffu, Llast, ((nb - 1) % KH) * GMAX + gl);
            }
            Mx = Mb;
            if constexpr (DET) {
                // 3. ||o||^2 before the batch, then fold the batch into this warp's slice
                float n2[2] = {0.f, 0.f};
#pragma unroll
                for (int i = 0; i < NVW; ++i)
#pragma unroll
                    for (int e = 0; e < VW; ++e) {
                        o0[i][e] = o[i][e];
                        n2[e & 1] = __fmaf_rn(o[i][e], o[i][e], n2[e & 1]);
                    }
                n0part = __fadd_rn(n2[0], n2[1]);
            }
            fold_batch(s0, nb - 1, beta, beta_hi, v, DET);
        }
        if constexpr (!DET) {
            // no detector: the merge warps agreed on the batch (or the failure)
            // before the fold; they meet once more so that no warp still reads
            // the batch's slots when they are handed back to the producers
            if (local_fail) {
                failed = true;
                break;
            }
            if constexpr (NM > 1)
                merge_barrier(NM * 32);
            else
                __syncwarp();
            if (mw == 0 && lane == 0)
                st_relaxed_cluster_u32(ctrl_cl, (uint32_t)(j0 + nb));
            j0 += nb;
            s0 += nb;
            if (s0 >= a.R) {
                s0 -= a.R;
                ph0 ^= 1u;
            }
            continue;
        }
        // 4. lane 2k+q (and 2k+q+16): sum over the warp of quantity q of batch block k
        reduce_scatter16(v, lane);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
            n0part += __shfl_xor_sync(0xffffffffu, n0part, off);
        // the slices meet; a failure anywhere ends the walk for every merge warp
        float *red = sh.red + (batch & 1) * (NM * 34);
        red[mw * 34 + lane] = v[0];
        if (lane == 0) {
            reinterpret_cast<volatile int *>(red)[mw * 34 + 32] = local_fail ? 1 : 0;
            red[mw * 34 + 33] = n0part;
        }
        if constexpr (NM > 1)
            merge_barrier(NM * 32);
        else
            __syncwarp();
        bool any_fail = false;
        float tot = 0.f, n0b = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NM; ++w2) {
            any_fail |= reinterpret_cast<volatile int *>(red)[w2 * 34 + 32] != 0;
            tot += red[w2 * 34 + (lane & 15)];
            n0b += red[w2 * 34 + 33];
        }
        if (any_fail) {
            failed = true;
            break;
        }
        // 5. statistics of batch block k in lane 2k: ||o_{j-1}||^2 by a prefix
        //    sum of t = 2 o_{j-1}.Delta + ||Delta||^2 over the batch's earlier
        //    blocks; the direction change uses the part of Delta orthogonal to
        //    o_{j-1}, so no near-equal O(1) numbers are subtracted.
        const float Dp = tot;
        const float Ep = __shfl_down_sync(0xffffffffu, tot, 1);
        const float t = 2.f * Dp + Ep;
        float pre = t;  // inclusive prefix over k in the even lanes 0..14
#pragma unroll
        for (int off = 2; off < 16; off <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, pre, off);
            if ((lane & 15) >= off)
                pre += u;
        }
        const float n0 = n0b + (pre - t);
        const float n1sq = n0 + t;
        bool stable = false;
        if (n0 > 0.f && n1sq > 0.f) {
            const float i0 = rsqrtf(n0), i1 = rsqrtf(n1sq);
            const float r0 = n0 * i0, r1 = n1sq * i1;
            const float d_scale = __fdividef(fabsf(t), (r1 + r0) * r0);
            const float pr = Dp * i0;  // component of Delta along o_{j-1}
            const float x = r0 + pr;
            const float y2 = fmaxf(fmaf(-pr, pr, Ep), 0.f);
            const float d_dir = x > 0.f ? __fdividef(y2, r1 * (r1 + x)) : fmaf(-x, i1, 1.f);
            stable = (d_scale < eps_m) && (d_dir < eps_d);
        }
        // 6. patience over the batch, one lane per block: the counter after
        //    block k is the run of stable blocks ending at k, plus the carried
        //    count when the run reaches back to the batch start.  Block j = 0
        //    of the walk is never compared, so it never counts as stable.
        const bool stab_k = __shfl_sync(0xffffffffu, stable, 2 * (lane & 7)) && (j0 + (lane & 7) >= 1);
        const uint32_t sbits = __ballot_sync(0xffffffffu, lane < nb && stab_k);
        const int kq = lane & 7;
        const uint32_t zeros = ~sbits & ((2u << kq) - 1u);  // unstable blocks at or before kq
        const int run = zeros == 0u ? cnt + kq + 1 : kq - (31 - __clz(zeros));
        const uint32_t hit = __ballot_sync(0xffffffffu, lane < nb && run >= P && j0 + kq + 1 >= minb);
        const int kstop = hit ? __ffs(hit) - 1 : -1;
        cnt = __shfl_sync(0xffffffffu, run, nb - 1);
        if (kstop >= 0) {
            stop = j0 + kstop + 1;
            if (kstop < nb - 1) {  // replay the batch up to the stop block
#pragma unroll
                for (int i = 0; i < NVW; ++i)
#pragma unroll
                    for (int e = 0; e < VW; ++e)
                        o[i][e] = o0[i][e];
                fold_batch(s0, kstop, beta, beta_hi, v, false);
            }
        }
        // Slots of this batch are free again (or the walk is over).  Every value
        // read from them has already fed the decision above, so a relaxed store
        // cannot overtake those reads.
        if (mw == 0 && lane == 0)
            st_relaxed_cluster_u32(ctrl_cl, stop ? (kStopBit | (uint32_t)stop) : (uint32_t)(j0 + nb));
        j0 += nb;
        s0 += nb;
        if (s0 >= a.R) {
            s0 -= a.R;
            ph0 ^= 1u;
        }
    }
    if (!failed && stop == 0)
        stop = N;
    if (failed && mw == 0 && lane == 0)
        st_relaxed_cluster_u32(ctrl_cl, kStopBit);
    float *op = a.out + (int64_t)b * a.out_sb;
#pragma unroll
    for (int ii = 0; ii < NVW; ++ii)
#pragma unroll
        for (int e = 0; e < VW; ++e) {
            const int i = vbase + ii;
            const int g = Lay::head(lane, i, e);
            const float val = o[ii][e];
            if (g < G && (Lay::kTwoHeads || i < G))
                op[(int64_t)(h * G + g) * a.out_sh + Lay::dim(lane, i, e)] = failed ? 0.f : val;
        }
    if (mw == 0 && lane == 0)
        a.stop_block[(int64_t)b * a.stop_sb + (int64_t)h * a.stop_sh] = failed ? -1 : stop;
}

// Several query tokens of one sequence sharing one walk: NQ tokens of GQ
// heads each, G = NQ * GQ rows in the block states.  The blocks are folded
// as in merge_role; what differs is that every token keeps its own
// statistics (over its own GQ * d outputs), patience counter and stop.  The
// sums of o.Delta, |Delta|^2 and |o|^2 are split by token, the patience rule
// runs once per token, and a token that has stopped is frozen: its rows get
// beta = 0 for every later block, so its output stays the prefix output at
// its own stop (a stop inside a batch replays the batch with the stopped
// token's later blocks weighted 0).  Each token's stop and output are those
// of its own single-query walk; the walk ends when every token has stopped.
// KB = 16 / NQ blocks per batch, so that the (block, token) sums fill the
// 32 lanes of one reduce-scatter.
template <int D, int GMAX, int ENGINE, int NMW, int NQ>
__device__ void merge_role_multi(const KernelArgs &a, const Shared &sh, int b, int h, int N, int mw)
{
    using MS = MergeShape<D, GMAX, ENGINE, NMW>;
    using Lay = typename MS::Lay;
    constexpr int NVW = MS::NVW, VW = Lay::VW, VP = VW / 2, NM = MS::NM;
    constexpr int KB = 16 / NQ;                  // blocks per batch
    constexpr int KH = 32 / GMAX;                // blocks per row of scan lanes
    constexpr int NH = KB > KH ? KB / KH : 1;    // (block, row) entries per scan lane
    constexpr int RS = 32 + 1 + NQ;              // exchange floats per merge warp: sums, flag, norms
    constexpr uint32_t ALL = (1u << NQ) - 1u;
    static_assert(NQ == 1 || NQ == 2 || NQ == 4, "tokens per walk");
    static_assert(NH * KH >= KB && NH <= 4, "scan rows");
    static_assert(2 * 4 * RS <= kRedFloats, "exchange buffer");
    const int lane = threadIdx.x & 31;
    const int G = a.G, GQ = a.GQ;
    const float eps_m = a.eps_m_arr ? a.eps_m_arr[b] : a.eps_m;
    const float eps_d = a.eps_d_arr ? a.eps_d_arr[b] : a.eps_d;
    const int P = a.P_arr ? a.P_arr[b] : a.P;
    const int minb = a.minb_arr ? a.minb_arr[b] : a.min_blocks;
    const uint32_t ctrl_cl = mapa(smem_u32((const void *)sh.ctrl), 0);
    const uint32_t u_off = sh.L.u_off_floats;
    const int slot_floats = (int)(sh.L.slot_bytes / 4);
    const int vbase = mw * NVW;

    // scan lane: blocks kl (and kl + KH) of the batch, row gl of token tok_gl
    const int kl = lane / GMAX, gl = lane % GMAX;
    const int tok_gl = gl < G ? gl / GQ : NQ;
    // token of the low and high half of each packed pair this lane keeps
    // (NQ for padding rows, which never count)
    int tlo[NVW], thi[NVW];
#pragma unroll
    for (int ii = 0; ii < NVW; ++ii) {
        const int r0 = Lay::head(lane, vbase + ii, 0), r1 = Lay::head(lane, vbase + ii, 1);
        tlo[ii] = r0 < G ? r0 / GQ : NQ;
        thi[ii] = r1 < G ? r1 / GQ : NQ;
    }
    float Mx = -CUDART_INF_F, Lm = 0.f;
    uint64_t o[NVW][VP];
#pragma unroll
    for (int i = 0; i < NVW; ++i)
#pragma unroll
        for (int q = 0; q < VP; ++q)
            o[i][q] = 0ull;

    int cnt[NQ], stop[NQ];
#pragma unroll
    for (int t = 0; t < NQ; ++t) {
        cnt[t] = 0;
        stop[t] = 0;
    }
    uint32_t done = 0u;  // bit t: token t has stopped (the same in every lane)
    bool failed = false;
    if (a.debug_flags & 1) {
        if (!warp_wait<true>(sh.never(), 0u, sh.abort, a.timeout_ns, a.device_status))
            failed = true;
    }

    auto load_u = [&](const float *sp, uint64_t (&uv)[NVW][VP]) {
#pragma unroll
        for (int ii = 0; ii < NVW; ++ii) {
            const float *up = sp + u_off + Lay::off(lane, vbase + ii);
            if constexpr (VW == 4) {
                const float4 x = *reinterpret_cast<const float4 *>(up);
                uv[ii][0] = pk2(x.x, x.y);
                uv[ii][1] = pk2(x.z, x.w);
            } else {
                const float2 x = *reinterpret_cast<const float2 *>(up);
                uv[ii][0] = pk2(x.x, x.y);
            }
        }
    };
    // split packed per-vector sums by token: entry t of out gets the halves of token t
    auto by_token = [&](const uint64_t (&x)[NVW], float (&out)[NQ]) {
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
            float acc = 0.f;
#pragma unroll
            for (int ii = 0; ii < NVW; ++ii) {
                acc += tlo[ii] == t ? lo2(x[ii]) : 0.f;
                acc += thi[ii] == t ? hi2(x[ii]) : 0.f;
            }
            out[t] = acc;
        }
    };
    // fold batch block k into this warp's slice; with sums, v[2 (k NQ + t)]
    // and v[2 (k NQ + t) + 1] get token t's o.Delta and |Delta|^2 of the slice
    auto fold = [&](int k, float beta, uint64_t bq, const uint64_t (&uv)[NVW][VP], float (&v)[32], bool sums) {
        uint64_t bp[NVW];
        const int kr = NH > 1 ? k % KH : k;
        if constexpr (Lay::kTwoHeads) {  // bq: the block's beta pair, fetched before the fold
#pragma unroll
            for (int ii = 0; ii < NVW; ++ii)
                bp[ii] = bq;
        } else {
#pragma unroll
            for (int ii = 0; ii < NVW; ++ii) {
                const float bi = __shfl_sync(0xffffffffu, beta, kr * GMAX + vbase + ii);
                bp[ii] = (vbase + ii < G) ? pk2(bi, bi) : 0ull;
            }
        }
        uint64_t sd[NVW], se[NVW];
#pragma unroll
        for (int ii = 0; ii < NVW; ++ii) {
            sd[ii] = 0ull;
            se[ii] = 0ull;
            if (!Lay::kTwoHeads && vbase + ii >= G)
                continue;  // padding rows: never written (see merge_role)
#pragma unroll
            for (int q = 0; q < VP; ++q) {
                // o += beta (u - o) as one fused step, as in merge_role
                const uint64_t df = sub2(uv[ii][q], o[ii][q]);
                if (sums) {
                    const uint64_t dl = mul2(bp[ii], df);
                    sd[ii] = fma2(o[ii][q], dl, sd[ii]);
                    se[ii] = fma2(dl, dl, se[ii]);
                }
                o[ii][q] = fma2(bp[ii], df, o[ii][q]);
            }
        }
        if (sums) {
            float pd[NQ], pe[NQ];
            by_token(sd, pd);
            by_token(se, pe);
#pragma unroll
            for (int t = 0; t < NQ; ++t) {
                v[2 * (k * NQ + t)] = pd[t];
                v[2 * (k * NQ + t) + 1] = pe[t];
            }
        }
    };
    auto fold_batch = [&](int s0, int kend, const float (&bh)[NH], float (&v)[32], bool sums) {
        uint64_t ua[NVW][VP], ub[NVW][VP];
        load_u(sh.ring + (size_t)s0 * slot_floats, ua);
        uint64_t bq[KB];  // as in merge_role: every block's beta pair before the fold
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            bq[k] = 0ull;
            if constexpr (Lay::kTwoHeads) {
                const int kr = NH > 1 ? k % KH : k;
                const int h0 = Lay::head(lane, 0, 0);
                bq[k] = pk2(__shfl_sync(0xffffffffu, bh[k / KH], kr * GMAX + h0),
                            __shfl_sync(0xffffffffu, bh[k / KH], kr * GMAX + h0 + 1));
            }
        }
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            if (k > kend)
                break;
            if (k + 1 <= kend) {
                int sn = s0 + k + 1;
                sn = sn >= a.R ? sn - a.R : sn;
                load_u(sh.ring + (size_t)sn * slot_floats, (k & 1) ? ua : ub);
            }
            fold(k, bh[k / KH], bq[k], (k & 1) ? ub : ua, v, sums);
        }
    };

    int s0 = 0;
    uint32_t ph0 = 0;
    for (int j0 = 0, batch = 0; !failed && done != ALL && j0 < N; ++batch) {
        const int nmax = min(KB, N - j0);
        // 1. wait for the batch (as in merge_role)
        int sk = s0 + (lane < KB ? lane : 0);
        uint32_t pk = ph0;
        if (sk >= a.R) {
            sk -= a.R;
            pk ^= 1u;
        }
        const float *spk = sh.ring + (size_t)sk * slot_floats;
        bool local_fail = false;
        int nb = 0;
        if (mw == 0) {
            uint64_t t0 = 0;
            for (uint32_t it = 0;; ++it) {
                const bool arrived = lane < nmax && mbar_try_wait(sh.ready(sk), pk);
                if (__any_sync(0xffffffffu, arrived && __float_as_uint(spk[0]) != 0u)) {
                    local_fail = true;
                    break;
                }
                if (__all_sync(0xffffffffu, arrived || lane >= nmax)) {
                    nb = nmax;
                    break;
                }
                if ((it & 7u) == 7u) {
                    int quit = 0;
                    if (lane == 0) {
                        const uint64_t now = global_timer_ns();
                        if (t0 == 0)
                            t0 = now;
                        if (*sh.abort) {
                            quit = 1;
                        } else if ((int64_t)(now - t0) > a.timeout_ns) {
                            *sh.abort = 1u;
                            record_error(a.device_status, kErrTimeout);
                            quit = 1;
                        }
                    }
                    if (__shfl_sync(0xffffffffu, quit, 0)) {
                        local_fail = true;
                        break;
                    }
                }
            }
        }
        if constexpr (NM > 1) {
            volatile int *agreed = reinterpret_cast<volatile int *>(sh.red + kRedFloats) + (batch & 1);
            if (mw == 0 && lane == 0)
                *agreed = local_fail ? -1 : nb;
            merge_barrier2(NM * 32);
            const int vv = *agreed;
            local_fail = vv < 0;
            nb = vv < 0 ? 0 : vv;
        }
        float v[32];
#pragma unroll
        for (int q = 0; q < 32; ++q)
            v[q] = 0.f;
        float bh[NH];  // beta of scan entry hh: block kl + hh KH, row gl
#pragma unroll
        for (int hh = 0; hh < NH; ++hh)
            bh[hh] = 0.f;
        float n0part[NQ];
#pragma unroll
        for (int t = 0; t < NQ; ++t)
            n0part[t] = 0.f;
        uint64_t o0[NVW][VP];
        if (!local_fail) {
            // 2. shares of the softmax mass per row; rows of stopped tokens get 0
            float mk[NH], lk[NH];
            float Mb = Mx;
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
                const int k = kl + hh * KH;
                mk[hh] = -CUDART_INF_F;
                lk[hh] = 0.f;
                if (k < nb && gl < G) {
                    int sl = s0 + k;
                    sl = sl >= a.R ? sl - a.R : sl;
                    const float *sp = sh.ring + (size_t)sl * slot_floats;
                    mk[hh] = sp[4 + gl];
                    lk[hh] = sp[4 + GMAX + gl];
                }
                Mb = fmaxf(Mb, mk[hh]);
            }
#pragma unroll
            for (int off = GMAX; off < 32; off <<= 1)
                Mb = fmaxf(Mb, __shfl_xor_sync(0xffffffffu, Mb, off));
            float w[NH], S[NH];
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
                w[hh] = (mk[hh] == -CUDART_INF_F) ? 0.f : __fmul_rn(lk[hh], ex2_approx(mk[hh] - Mb));
                S[hh] = w[hh];
            }
#pragma unroll
            for (int off = GMAX; off < 32; off <<= 1)
#pragma unroll
                for (int hh = 0; hh < NH; ++hh) {
                    const float t = __shfl_up_sync(0xffffffffu, S[hh], off);
                    if (lane >= off)
                        S[hh] += t;
                }
            // each row of scan lanes continues from the total of the rows before it
            float carry = 0.f;
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
                S[hh] += carry;
                if (hh + 1 < NH)
                    carry = __shfl_sync(0xffffffffu, S[hh], (KH - 1) * GMAX + gl);
            }
            const float base = (Mx == -CUDART_INF_F) ? 0.f : __fmul_rn(Lm, ex2_approx(Mx - Mb));
            const bool frozen = tok_gl < NQ && ((done >> tok_gl) & 1u);
            float Lam[NH];
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
                Lam[hh] = base + S[hh];
                bh[hh] = (Lam[hh] > 0.f && !frozen) ? __fmul_rn(w[hh], rcp_approx(Lam[hh])) : 0.f;
            }
            const int hl = (nb - 1) / KH;  // row of the batch's last block
            float Llast = Lam[0];
#pragma unroll
            for (int hh = 1; hh < NH; ++hh)
                Llast = hl == hh ? Lam[hh] : Llast;
            Lm = __shfl_sync(0xffffffffu, Llast, ((nb - 1) % KH) * GMAX + gl);
            Mx = Mb;
            // 3. per-token ||o||^2 before the batch, then fold the batch
            uint64_t n2[NVW];
#pragma unroll
            for (int i = 0; i < NVW; ++i) {
                n2[i] = 0ull;
#pragma unroll
                for (int q = 0; q < VP; ++q) {
                    o0[i][q] = o[i][q];
                    n2[i] = fma2(o[i][q], o[i][q], n2[i]);
                }
            }
            by_token(n2, n0part);
            fold_batch(s0, nb - 1, bh, v, true);
        }
        // 4. lane l: warp sum of entry l = 2 (k NQ + t) + q
        reduce_scatter32(v, lane);
#pragma unroll
        for (int t = 0; t < NQ; ++t)
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
                n0part[t] += __shfl_xor_sync(0xffffffffu, n0part[t], off);
        float *red = sh.red + (batch & 1) * (NM * RS);
        red[mw * RS + lane] = v[0];
        if (lane == 0) {
            reinterpret_cast<volatile int *>(red)[mw * RS + 32] = local_fail ? 1 : 0;
#pragma unroll
            for (int t = 0; t < NQ; ++t)
                red[mw * RS + 33 + t] = n0part[t];
        }
        if constexpr (NM > 1)
            merge_barrier(NM * 32);
        else
            __syncwarp();
        bool any_fail = false;
        float tot = 0.f, n0b[NQ];
#pragma unroll
        for (int t = 0; t < NQ; ++t)
            n0b[t] = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NM; ++w2) {
            any_fail |= reinterpret_cast<volatile int *>(red)[w2 * RS + 32] != 0;
            tot += red[w2 * RS + lane];
#pragma unroll
            for (int t = 0; t < NQ; ++t)
                n0b[t] += red[w2 * RS + 33 + t];
        }
        if (any_fail) {
            failed = true;
            break;
        }
        // 5. statistics of (block k, token t) in lane 2 (k NQ + t); the prefix
        //    over k of token t runs over lanes 2 NQ apart
        const int tl = (lane >> 1) % NQ;
        const float Dp = tot;
        const float Ep = __shfl_down_sync(0xffffffffu, tot, 1);
        const float tt = 2.f * Dp + Ep;
        float pre = tt;
#pragma unroll
        for (int off = 2 * NQ; off < 32; off <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, pre, off);
            if (lane >= off)
                pre += u;
        }
        float n0base = n0b[0];
#pragma unroll
        for (int t = 1; t < NQ; ++t)
            n0base = tl == t ? n0b[t] : n0base;
        const float n0 = n0base + (pre - tt);
        const float n1sq = n0 + tt;
        bool stable = false;
        if (n0 > 0.f && n1sq > 0.f) {
            const float i0 = rsqrtf(n0), i1 = rsqrtf(n1sq);
            const float r0 = n0 * i0, r1 = n1sq * i1;
            const float d_scale = __fdividef(fabsf(tt), (r1 + r0) * r0);
            const float pr = Dp * i0;
            const float x = r0 + pr;
            const float y2 = fmaxf(fmaf(-pr, pr, Ep), 0.f);
            const float d_dir = x > 0.f ? __fdividef(y2, r1 * (r1 + x)) : fmaf(-x, i1, 1.f);
            stable = (d_scale < eps_m) && (d_dir < eps_d);
        }
        // 6. patience per token, one lane per block (as in merge_role)
        const int kq = lane & (KB - 1);
        int kstop[NQ];
        bool replay = false;
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
            const bool stab_k = __shfl_sync(0xffffffffu, stable, 2 * (kq * NQ + t)) && (j0 + kq >= 1);
            const uint32_t sbits = __ballot_sync(0xffffffffu, lane < nb && stab_k);
            const uint32_t zeros = ~sbits & ((2u << kq) - 1u);
            const int run = zeros == 0u ? cnt[t] + kq + 1 : kq - (31 - __clz(zeros));
            const uint32_t hit = __ballot_sync(0xffffffffu, lane < nb && run >= P && j0 + kq + 1 >= minb);
            const int run_last = __shfl_sync(0xffffffffu, run, nb - 1);
            kstop[t] = -1;
            if (!((done >> t) & 1u)) {
                cnt[t] = run_last;
                if (hit) {
                    kstop[t] = __ffs(hit) - 1;
                    stop[t] = j0 + kstop[t] + 1;
                    replay |= kstop[t] < nb - 1;
                }
            }
        }
        if (replay) {
            // fold the batch again from the snapshot, each token that stopped
            // inside it weighted 0 after its stop block
#pragma unroll
            for (int i = 0; i < NVW; ++i)
#pragma unroll
                for (int q = 0; q < VP; ++q)
                    o[i][q] = o0[i][q];
            int ks = NQ > 0 ? kstop[0] : -1;
#pragma unroll
            for (int t = 1; t < NQ; ++t)
                ks = tok_gl == t ? kstop[t] : ks;
            if (tok_gl < NQ && ks >= 0) {
#pragma unroll
                for (int hh = 0; hh < NH; ++hh)
                    if (kl + hh * KH > ks)
                        bh[hh] = 0.f;
            }
            fold_batch(s0, nb - 1, bh, v, false);
        }
        int maxstop = 0;
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
            if (kstop[t] >= 0)
                done |= 1u << t;
            maxstop = max(maxstop, stop[t]);
        }
        if (mw == 0 && lane == 0)
            st_relaxed_cluster_u32(ctrl_cl, done == ALL ? (kStopBit | (uint32_t)maxstop) : (uint32_t)(j0 + nb));
        j0 += nb;
        s0 += nb;
        if (s0 >= a.R) {
            s0 -= a.R;
            ph0 ^= 1u;
        }
    }
    if (!failed) {
#pragma unroll
        for (int t = 0; t < NQ; ++t)
            if (!((done >> t) & 1u))
                stop[t] = N;
    }
    if (failed && mw == 0 && lane == 0)
        st_relaxed_cluster_u32(ctrl_cl, kStopBit);
    float *op = a.out + (int64_t)b * a.out_sb;
#pragma unroll
    for (int ii = 0; ii < NVW; ++ii)
#pragma unroll
        for (int e = 0; e < VW; ++e) {
            const int i = vbase + ii;
            const int r = Lay::head(lane, i, e);
            const float val = (e & 1) ? hi2(o[ii][e >> 1]) : lo2(o[ii][e >> 1]);
            if (r < G && (Lay::kTwoHeads || i < G)) {
                const int t = r / GQ, g = r - t * GQ;
                op[(int64_t)t * a.out_st + (int64_t)(h * GQ + g) * a.out_sh + Lay::dim(lane, i, e)] =
                    failed ? 0.f : val;
            }
        }
    if (mw == 0) {
#pragma unroll
        for (int t = 0; t < NQ; ++t)
            if (lane == t)
                a.stop_block[(int64_t)b * a.stop_sb + (int64_t)t * a.stop_st + (int64_t)h * a.stop_sh] =
                    failed ? -1 : stop[t];
    }
}

// ---- kernel ------------------------------------------------------------------------

// NQ: query tokens sharing the walk (1: merge_role, else merge_role_multi).
// DET: false for the single-query walk without the detector (see merge_role).
// (the shared walks with one merge warp launch at most eight warps: their
// bound leaves them the registers the two-token merge needs)
template <typename T, int D, int PAGE, int GMAX, int ENGINE, int NMW, int NQ = 1, bool DET = true>
__global__ void __launch_bounds__((NQ > 1 && NMW == 1) ? 256 : kMaxThreads, 1)
    art_walk_kernel(const KernelArgs a, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    Shared sh;
    sh.L = make_layout(a.S, a.NW, a.R, PAGE, D, (int)sizeof(T), GMAX, ENGINE != kEngineMma);
    sh.kv = base + sh.L.kv_off;
    sh.ring = reinterpret_cast<float *>(base + sh.L.ring_off);
    sh.pbuf = reinterpret_cast<float *>(base + sh.L.pbuf_off);
    sh.red = reinterpret_cast<float *>(base + sh.L.red_off);
    sh.stage_j = reinterpret_cast<uint32_t *>(base + sh.L.meta_off);
    sh.stage_nv = sh.stage_j + a.S;
    const uint32_t bar0 = smem_u32(base + sh.L.bar_off);
    sh.bar_full_k = bar0;
    sh.bar_full_v = bar0 + 8u * a.S;
    sh.bar_empty = bar0 + 16u * a.S;
    sh.bar_ready = bar0 + 24u * a.S;
    sh.bar_never = bar0 + 8u * (3 * a.S + a.R);
    sh.ring_leader = smem_u32(sh.ring);
    sh.ready_leader = sh.bar_ready;
    sh.ctrl = reinterpret_cast<volatile uint32_t *>(base + sh.L.ctrl_off);
    sh.fetched = sh.ctrl + 1;
    sh.abort = sh.ctrl + 2;

    const int warp = threadIdx.x >> 5;
    const uint32_t rank = cluster_ctarank();
    const int unit = blockIdx.x / a.C;
    const int b = unit / a.Hkv, h = unit % a.Hkv;
    const int Lseq = a.seq_lens[b];
    // (written so that lengths near INT32_MAX do not overflow: they are
    // longer than any page table and reported below)
    const int N = Lseq <= 0 ? 0 : Lseq / PAGE + (Lseq % PAGE != 0);
    const bool bad_len = N > a.max_blocks;

    constexpr int NM = MergeShape<D, GMAX, ENGINE, NMW>::NM;
    const bool walk = N > 0 && !bad_len;
    // Start the first global reads now, so that they are in flight during the
    // set-up barriers: the producer's first 32 (block, page) pairs, the compute
    // warps' queries.
    int first_lb = -1, first_pp = -1;
    if (walk && warp == 0) {
        const int jj = (int)rank + (threadIdx.x & 31) * a.C;
        if (jj < N)
            // no order given: the sink block, then newest to oldest
            first_lb = a.block_order ? __ldg(a.block_order + (int64_t)b * a.bo_sb + jj) : (jj == 0 ? 0 : N - jj);
    }
    EngineFor<T, D, PAGE, GMAX, ENGINE> eng;
    if (walk && warp > NM) {
        if constexpr (NQ == 1)
            eng.load_q(a, b, h, threadIdx.x & 31);
        else
            eng.load_q_rows(a, b, h, threadIdx.x & 31);
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.S; ++s) {
            mbar_init(sh.full_k(s), 1);
            mbar_init(sh.full_v(s), 1);
            mbar_init(sh.empty(s), 1);
        }
        for (int r = 0; r < a.R; ++r)
            mbar_init(sh.ready(r), 1);
        mbar_init(sh.never(), 1);
        sh.ctrl[0] = 0u;
        sh.ctrl[1] = 0u;
        sh.ctrl[2] = 0u;
        fence_mbar_init_cluster();
    }
    __syncthreads();
    if (walk && warp == 0 && first_lb >= 0 && first_lb < N)
        first_pp = __ldg(a.page_table + (int64_t)b * a.pt_sb + first_lb);
    cluster_sync();  // remote CTAs may now arrive on the leader's barriers

    if (walk) {
        if (warp == 0)
            producer_role<T, D, PAGE, ENGINE>(a, sh, &tmk, &tmv, b, h, N, Lseq, rank, a.C, first_lb, first_pp);
        else if (warp <= NM) {
            if (rank == 0) {
                if constexpr (NQ == 1)
                    merge_role<D, GMAX, ENGINE, NMW, DET>(a, sh, b, h, N, warp - 1);
                else
                    merge_role_multi<D, GMAX, ENGINE, NMW, NQ>(a, sh, b, h, N, warp - 1);
            }
        } else
            compute_role<T, D, PAGE, GMAX, ENGINE>(a, sh, b, h, warp - 1 - NM, eng);
    } else if (rank == 0 && warp == 1) {
        const int lane = threadIdx.x & 31;
        float *op = a.out + (int64_t)b * a.out_sb;
        if constexpr (NQ == 1) {
            for (int i = lane; i < a.G * D; i += 32)
                op[(int64_t)(h * a.G + i / D) * a.out_sh + i % D] = 0.f;
        } else {
            for (int i = lane; i < a.G * D; i += 32) {
                const int r = i / D, t = r / a.GQ, g = r - t * a.GQ;
                op[(int64_t)t * a.out_st + (int64_t)(h * a.GQ + g) * a.out_sh + i % D] = 0.f;
            }
        }
        if (lane < NQ)
            a.stop_block[(int64_t)b * a.stop_sb + (int64_t)lane * a.stop_st + (int64_t)h * a.stop_sh] =
                bad_len ? -1 : 0;
        if (lane == 0 && bad_len)
            record_error(a.device_status, kErrBadIndex);
    }
    __syncwarp();
    cluster_sync();  // remote stores into the leader are complete
    if (rank == 0 && threadIdx.x == 0 && a.blocks_fetched)
        a.blocks_fetched[unit] = (int32_t)sh.fetched[0];
}

}  // namespace art
