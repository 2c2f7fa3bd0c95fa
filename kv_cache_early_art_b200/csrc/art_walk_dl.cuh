// art_walk_dl.cuh -- the ART walk with a dedicated merge CTA, for launches
// with few (sequence, kv-head) units spread over large clusters.
//
// Method as in art_kernels.cuh ("ART: Attention Run-time Termination for
// Efficient Large Language Model Decoding", gist.science explainer, Technical
// Summary 2.1-2.4).  What differs is how the work is laid out over a cluster
// of C CTAs serving one unit:
//
//   rank 0 (merge CTA)   holds the state ring (its whole shared memory, so the
//                        speculation window is deep) and runs the merge in
//                        three stages that overlap across batches:
//                          share warp   polls the batch and forms the blocks'
//                                       shares of the softmax mass;
//                          fold warps   (NMF of them, the head dimension split
//                                       over them) fold the batch into the
//                                       running output and reduce their
//                                       slices' sums (o.Delta, |Delta|^2,
//                                       |o|^2 per block);
//                          decision warp takes the sums of a batch, forms the
//                                       two statistics, runs the patience rule
//                                       and publishes the merged count (or the
//                                       stop) to the producers,
//                        so the shares of batch b + 1 are formed while batch b
//                        is folded, and batch b + 1 is folded while batch b is
//                        being decided.  The stages hand over through
//                        mbarrier-guarded two-entry rings.  They keep at most two undecided
//                        batches, with a snapshot of the output at the start
//                        of each, and a stop inside one of them replays it up
//                        to the stop: stop and output are those of a strictly
//                        sequential walk, as in merge_role.
//   ranks 1 .. C-1       fetch and compute: producer warp and compute warps
//                        exactly as in art_walk_kernel, with steps
//                        j = rank - 1, rank - 1 + (C - 1), ... and every block
//                        state pushed into the merge CTA's ring.
//
// The slots of a batch are handed back to the producers only once its
// decision is made, so a replay always finds the states it needs.
#pragma once

#include "art_kernels.cuh"

namespace art {

// Exchange area of the dedicated merge (floats): two batches of fold-warp
// sums (up to eight warps x 32 sums, the batch size, the norm), two batches
// of shares (block k, head g at k * 8 + g, the batch size at 64), then the
// control words.
constexpr int kDLSumFloats = 2 * 8 * 34;
constexpr int kDLBetaFloats = 8 * 8 + 4;
constexpr int kDLCtlOff = kDLSumFloats + 2 * kDLBetaFloats;
constexpr int kDLRedFloats = kDLCtlOff + 16;
constexpr int kDLNone = 0x7fffffff;  // no final decision published yet
constexpr int kDLFailed = -1;
constexpr int kDLBars = 10;          // sums_full[2], beta_full[2], beta_empty[2], dec[2], landed[2]

// Shared-memory carve-up.  The control words and the state ring's ready
// barriers sit at the same offsets in every CTA of the cluster, so the workers
// reach the merge CTA's with mapa:
//   [0, 16)              ctrl (merged count / stop), fetched, abort, pad
//   [16, 16 + 8 (R + 1)) ready[R], never
//   bar_off              full_k[S], full_v[S], empty[S], then the merge's
//                        sums_full[2], beta_full[2], beta_empty[2], dec[2]
//   meta_off             stage_j[S], stage_nv[S]
//   red_off              kDLRedFloats floats
//   kv_off (1024-align)  S stages of [K tile | V tile]          (workers)
//   ring_off             ring_slots block-state slots            (merge CTA)
struct DLLayout {
    uint32_t tile_bytes, stage_bytes, slot_bytes, u_off_floats;
    uint32_t bar_off, meta_off, red_off, kv_off, ring_off, total;
};

__host__ __device__ inline DLLayout make_dl_layout(int S, int R, int page, int d, int esize, int gmax, int ring_slots)
{
    DLLayout L;
    L.tile_bytes = (uint32_t)(page * d * esize);
    L.stage_bytes = 2 * L.tile_bytes;
    L.u_off_floats = round_up_u32(4 + 2 * gmax, 4);
    L.slot_bytes = round_up_u32((L.u_off_floats + gmax * d) * 4, 16);
    uint32_t off = 16 + 8 * (uint32_t)(R + 1);
    L.bar_off = off;
    off += 8 * (uint32_t)(3 * S + kDLBars);
    L.meta_off = off;
    off += 2 * (uint32_t)S * 4;
    off = round_up_u32(off, 16);
    L.red_off = off;
    off += kDLRedFloats * 4;
    off = round_up_u32(off, 1024);
    L.kv_off = off;
    off += (uint32_t)S * L.stage_bytes;
    L.ring_off = off;
    off += (uint32_t)ring_slots * L.slot_bytes;
    L.total = off;
    return L;
}

// The merge's mbarriers (shared addresses), two of each kind, by batch parity.
struct DLBars {
    uint32_t sums_full;   // the fold warps' sums of a batch are written (count NMF)
    uint32_t beta_full;   // the shares of a batch are written (count 1)
    uint32_t beta_empty;  // the fold warps have read them (count NMF)
    uint32_t dec;         // the decision warp has decided a batch (count 1)
    uint32_t landed;      // a batch's states have been copied in from the workspace (count 1)
};

// Bounded wait of a whole warp until pred() holds for lane 0's view.
// Returns false on abort or timeout (the latter raises abort and records the
// error).
template <typename Pred>
__device__ __forceinline__ bool warp_spin(Pred pred, volatile uint32_t *abort, int64_t timeout_ns, int32_t *status)
{
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        int v = 0;
        if ((threadIdx.x & 31) == 0) {
            if (pred()) {
                v = 1;
            } else if ((it & 15u) == 15u) {
                const uint64_t now = global_timer_ns();
                if (t0 == 0)
                    t0 = now;
                if (*abort) {
                    v = -1;
                } else if ((int64_t)(now - t0) > timeout_ns) {
                    *abort = 1u;
                    record_error(status, kErrTimeout);
                    v = -1;
                }
            }
        }
        v = __shfl_sync(0xffffffffu, v, 0);
        if (v != 0)
            return v > 0;
    }
}

__device__ __forceinline__ int ld_acquire_cta_s32(const volatile int *p)
{
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32((const void *)p)) : "memory");
    return v;
}

// ---- share warp ------------------------------------------------------------------

// Polls each batch's block states, forms the blocks' shares of the softmax
// mass (the scan of merge_role, step 2) and hands them to the fold warps
// through a two-entry ring: entry batch & 1, block k, head g at k * 8 + g,
// the batch size (or -1 on a failure, -2 once the final decision is in and
// the batch will never come) at 64.
template <int D, int GMAX, int ENGINE, int NMF>
__device__ void share_role_dl(const KernelArgs &a, const Shared &sh, int N, const DLBars &bars)
{
    using MS = MergeShape<D, GMAX, ENGINE, NMF>;
    constexpr int KB = MS::KB, KH = MS::KH, NH = MS::NH;
    const int lane = threadIdx.x & 31;
    const int G = a.G;
    const int slot_floats = (int)(sh.L.slot_bytes / 4);
    volatile int *ctl = reinterpret_cast<volatile int *>(sh.red + kDLCtlOff);
    const int kl = lane / GMAX, gl = lane % GMAX;
    float Mx = -CUDART_INF_F, Lm = 0.f;

    int s0 = 0;
    uint32_t ph0 = 0;
    for (int j0 = 0, batch = 0; j0 < N; ++batch) {
        const int e = batch & 1;
        float *be = sh.red + kDLSumFloats + e * kDLBetaFloats;
        int quit = 0;  // 1 failure, 2 final decision in
        if (batch >= 2) {
            // the entry is free once the fold warps have read batch b - 2; after
            // a stop they may never read it, so the final word also ends the wait
            const uint32_t bar = bars.beta_empty + 8u * e, par = (uint32_t)((batch - 2) >> 1) & 1u;
            if (!warp_spin([&] { return mbar_try_wait(bar, par) || ctl[3] != kDLNone; }, sh.abort, a.timeout_ns,
                           a.device_status))
                quit = 1;
            else if (!mbar_try_wait(bar, par))
                quit = 2;
            quit = __shfl_sync(0xffffffffu, quit, 0);
            __syncwarp();
        }
        const int nmax = min(KB, N - j0);
        int sk = s0 + (lane < KB ? lane : 0);
        uint32_t pk = ph0;
        if (sk >= a.R) {
            sk -= a.R;
            pk ^= 1u;
        }
        const float *spk = sh.ring + (size_t)sk * slot_floats;
        uint64_t t0 = 0;
        for (uint32_t it = 0; !quit; ++it) {
            // Once the final decision is in, the batch may never come, and a
            // try_wait on a phase that never completes suspends the warp until
            // the hardware's time limit: the final word is read before every
            // poll, so the warp leaves after at most one such suspension.
            if (__shfl_sync(0xffffffffu, lane == 0 && ctl[3] != kDLNone ? 1 : 0, 0)) {
                quit = 2;
                break;
            }
            const bool arrived = lane < nmax && mbar_try_wait(sh.ready(sk), pk);
            if (__any_sync(0xffffffffu, arrived && __float_as_uint(spk[0]) != 0u)) {
                quit = 1;
                break;
            }
            if (__all_sync(0xffffffffu, arrived || lane >= nmax))
                break;
            if ((it & 7u) == 7u) {
                int q = 0;
                if (lane == 0) {
                    const uint64_t now = global_timer_ns();
                    if (t0 == 0)
                        t0 = now;
                    if (*sh.abort) {
                        q = 1;
                    } else if ((int64_t)(now - t0) > a.timeout_ns) {
                        *sh.abort = 1u;
                        record_error(a.device_status, kErrTimeout);
                        q = 1;
                    }
                }
                quit = __shfl_sync(0xffffffffu, q, 0);
            }
        }
        if (quit) {
            if (lane == 0)
                reinterpret_cast<volatile int *>(be)[64] = quit == 1 ? -1 : -2;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bars.beta_full + 8u * e);
            break;
        }
        const int nb = nmax;
        // shares of the softmax mass: beta_(k,g) = w_k / (L_prev + w_0 + ... + w_k)
        float Mb = Mx;
        float mk[NH], lk[NH];
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
        float Lam[NH];
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
            Lam[hh] = base + S[hh];
            const float bt = Lam[hh] > 0.f ? __fmul_rn(w[hh], rcp_approx(Lam[hh])) : 0.f;
            const int k = kl + hh * KH;
            if (k < KB)
                be[k * 8 + gl] = bt;
        }
        const float Llast = (NH > 1 && nb - 1 >= KH) ? Lam[NH - 1] : Lam[0];
        Lm = __shfl_sync(0xffffffffu, Llast, ((nb - 1) % KH) * GMAX + gl);
        Mx = Mb;
        if (lane == 0)
            reinterpret_cast<volatile int *>(be)[64] = nb;
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bars.beta_full + 8u * e);
        j0 += nb;
        s0 += nb;
        if (s0 >= a.R) {
            s0 -= a.R;
            ph0 ^= 1u;
        }
    }
}

// ---- fold warps ------------------------------------------------------------------

// ctl[3]: the final decision (stop index, N at the end of the walk, kDLFailed)
// or kDLNone.
template <int D, int GMAX, int ENGINE, int NMF, bool DET>
__device__ void fold_role_dl(const KernelArgs &a, const Shared &sh, int b, int h, int N, int mw, const DLBars &bars)
{
    using MS = MergeShape<D, GMAX, ENGINE, NMF>;
    using Lay = typename MS::Lay;
    constexpr int NVW = MS::NVW, VW = Lay::VW, KB = MS::KB, NM = MS::NM;
    static_assert(NM == NMF, "one fold warp per slice");
    static_assert(KB <= 8 && NM <= 8 && GMAX <= 8, "exchange layout");
    static_assert(Lay::kTwoHeads, "the dedicated merge is built for the tensor-core state layout");
    const int lane = threadIdx.x & 31;
    const int G = a.G;
    const uint32_t u_off = sh.L.u_off_floats;
    const int slot_floats = (int)(sh.L.slot_bytes / 4);
    const int vbase = mw * NVW;
    const int h0 = Lay::head(lane, 0, 0);  // the lane's elements alternate between heads h0 and h0 + 1
    volatile int *ctl = reinterpret_cast<volatile int *>(sh.red + kDLCtlOff);

    float o[NVW][VW];
#pragma unroll
    for (int i = 0; i < NVW; ++i)
#pragma unroll
        for (int e = 0; e < VW; ++e)
            o[i][e] = 0.f;

    auto load_u = [&](const float *sp, float (&uv)[NVW][VW]) {
#pragma unroll
        for (int ii = 0; ii < NVW; ++ii) {
            const float4 x = *reinterpret_cast<const float4 *>(sp + u_off + Lay::off(lane, vbase + ii));
            uv[ii][0] = x.x;
            uv[ii][1] = x.y;
            uv[ii][2] = x.z;
            uv[ii][3] = x.w;
        }
    };
    // the fold of merge_role: o += beta (u - o) in one fused step, with the
    // slice's o.Delta and |Delta|^2 (even and odd elements apart, then added)
    auto fold_batch = [&](int s0, int kend, const float (&b0)[KB], const float (&b1)[KB], float (&v)[16], bool sums) {
        float ua[NVW][VW], ub[NVW][VW];
        load_u(sh.ring + (size_t)s0 * slot_floats, ua);
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            if (k > kend)
                break;
            if (k + 1 <= kend) {
                int sn = s0 + k + 1;
                sn = sn >= a.R ? sn - a.R : sn;
                load_u(sh.ring + (size_t)sn * slot_floats, (k & 1) ? ua : ub);
            }
            const float (&uv)[NVW][VW] = (k & 1) ? ub : ua;
            float sd[2] = {0.f, 0.f}, se[2] = {0.f, 0.f};
#pragma unroll
            for (int ii = 0; ii < NVW; ++ii)
#pragma unroll
                for (int e = 0; e < VW; ++e) {
                    const float bb = (e & 1) ? b1[k] : b0[k];
                    const float df = __fsub_rn(uv[ii][e], o[ii][e]);
                    if (sums) {
                        const float dl = __fmul_rn(bb, df);
                        sd[e & 1] = __fmaf_rn(o[ii][e], dl, sd[e & 1]);
                        se[e & 1] = __fmaf_rn(dl, dl, se[e & 1]);
                    }
                    o[ii][e] = __fmaf_rn(bb, df, o[ii][e]);
                }
            if (sums) {
                v[2 * k] = __fadd_rn(sd[0], sd[1]);
                v[2 * k + 1] = __fadd_rn(se[0], se[1]);
            }
        }
    };

    // the last two folded batches: output at their start, first slot, first
    // block, size and shares (P: the older, C: the newer)
    float oP[NVW][VW], oC[NVW][VW];
    float bP0[KB], bP1[KB], bC0[KB], bC1[KB];
    int s0P = 0, j0P = 0, nbP = 0, s0C = 0, j0C = 0, nbC = 0;
#pragma unroll
    for (int i = 0; i < NVW; ++i)
#pragma unroll
        for (int e = 0; e < VW; ++e)
            oP[i][e] = oC[i][e] = 0.f;
#pragma unroll
    for (int k = 0; k < KB; ++k)
        bP0[k] = bP1[k] = bC0[k] = bC1[k] = 0.f;

    bool failed = false;
    int s0 = 0, j0 = 0, batch = 0;
    while (j0 < N) {
        const int e = batch & 1;
        // 0. at most two batches ahead of the decisions: batch b starts once
        //    batch b - 2 is decided (and was not the stop)
        if (batch >= 2) {
            if (!warp_wait<false>(bars.dec + 8u * e, (uint32_t)((batch - 2) >> 1) & 1u, sh.abort, a.timeout_ns,
                                  a.device_status)) {
                failed = true;
                break;
            }
            if (ctl[3] != kDLNone)
                break;  // a stop inside the last two batches, or a failure
        }
        // 1. the batch's shares
        if (!warp_wait<false>(bars.beta_full + 8u * e, (uint32_t)(batch >> 1) & 1u, sh.abort, a.timeout_ns,
                              a.device_status)) {
            failed = true;
            break;
        }
        const float *be = sh.red + kDLSumFloats + e * kDLBetaFloats;
        const int nb = reinterpret_cast<const volatile int *>(be)[64];
        float *red = sh.red + e * (NM * 34);
        if (nb == -2)
            break;  // the final word is in: this batch will never come
        if (nb < 0) {
            // hand the failure to the decision warp
            if (lane == 0)
                reinterpret_cast<volatile int *>(red)[mw * 34 + 32] = -1;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bars.sums_full + 8u * e);
            failed = true;
            break;
        }
        // 2. snapshots of the last two batches, this batch's shares
#pragma unroll
        for (int i = 0; i < NVW; ++i)
#pragma unroll
            for (int q = 0; q < VW; ++q) {
                oP[i][q] = oC[i][q];
                oC[i][q] = o[i][q];
            }
#pragma unroll
        for (int k = 0; k < KB; ++k) {
            bP0[k] = bC0[k];
            bP1[k] = bC1[k];
            const float2 bt = *reinterpret_cast<const float2 *>(be + k * 8 + h0);
            bC0[k] = k < nb ? bt.x : 0.f;
            bC1[k] = k < nb ? bt.y : 0.f;
        }
        s0P = s0C; j0P = j0C; nbP = nbC;
        s0C = s0; j0C = j0; nbC = nb;
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bars.beta_empty + 8u * e);
        // 3. fold, and the slice's sums for the decision warp
        float v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q)
            v[q] = 0.f;
        float n0part = 0.f;
        if constexpr (DET) {
            float n2[2] = {0.f, 0.f};
#pragma unroll
            for (int i = 0; i < NVW; ++i)
#pragma unroll
                for (int q = 0; q < VW; ++q)
                    n2[q & 1] = __fmaf_rn(o[i][q], o[i][q], n2[q & 1]);
            n0part = __fadd_rn(n2[0], n2[1]);
        }
        fold_batch(s0, nb - 1, bC0, bC1, v, DET);
        if constexpr (DET) {
            reduce_scatter16(v, lane);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
                n0part += __shfl_xor_sync(0xffffffffu, n0part, off);
            red[mw * 34 + lane] = v[0];
            if (lane == 0)
                red[mw * 34 + 33] = n0part;
        }
        if (lane == 0)
            reinterpret_cast<volatile int *>(red)[mw * 34 + 32] = nb;
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bars.sums_full + 8u * e);
        j0 += nb;
        s0 += nb;
        if (s0 >= a.R)
            s0 -= a.R;
        ++batch;
    }
    // 4. the final decision
    int fin = kDLFailed;
    if (warp_spin([&] { return ctl[3] != kDLNone; }, sh.abort, a.timeout_ns, a.device_status))
        fin = ld_acquire_cta_s32(ctl + 3);
    if (fin == kDLFailed)
        failed = true;
    if (!failed && fin < j0) {
        // the stop lies in one of the last two folded batches: restart from
        // the snapshot of its batch and fold up to it
        const int last = fin - 1;
        float v[16];
        if (last >= j0C && last < j0C + nbC) {
#pragma unroll
            for (int i = 0; i < NVW; ++i)
#pragma unroll
                for (int q = 0; q < VW; ++q)
                    o[i][q] = oC[i][q];
            fold_batch(s0C, last - j0C, bC0, bC1, v, false);
        } else if (last >= j0P && last < j0P + nbP) {
#pragma unroll
            for (int i = 0; i < NVW; ++i)
#pragma unroll
                for (int q = 0; q < VW; ++q)
                    o[i][q] = oP[i][q];
            fold_batch(s0P, last - j0P, bP0, bP1, v, false);
        } else {
            failed = true;  // cannot happen: a stop is never decided outside the last two batches
        }
    }
    float *op = a.out + (int64_t)b * a.out_sb;
#pragma unroll
    for (int ii = 0; ii < NVW; ++ii)
#pragma unroll
        for (int q = 0; q < VW; ++q) {
            const int i = vbase + ii;
            const int g = Lay::head(lane, i, q);
            if (g < G)
                op[(int64_t)(h * G + g) * a.out_sh + Lay::dim(lane, i, q)] = failed ? 0.f : o[ii][q];
        }
}

// ---- decision warp ----------------------------------------------------------------

// GM: publish the merged count and the stop in the workspace (the fetching
// CTAs are not in this CTA's cluster) instead of this CTA's shared memory.
template <int D, int GMAX, int ENGINE, int NMF, bool DET, bool GM = false>
__device__ void decide_role_dl(const KernelArgs &a, const Shared &sh, int b, int h, int N, const DLBars &bars)
{
    const unsigned long long ep = (unsigned long long)a.epoch << 32;
    unsigned long long *gctrl = GM ? a.g_ctrl + (b * a.Hkv + h) : nullptr;
    const int lane = threadIdx.x & 31;
    const float eps_m = a.eps_m_arr ? a.eps_m_arr[b] : a.eps_m;
    const float eps_d = a.eps_d_arr ? a.eps_d_arr[b] : a.eps_d;
    const int P = a.P_arr ? a.P_arr[b] : a.P;
    const int minb = a.minb_arr ? a.minb_arr[b] : a.min_blocks;
    const uint32_t ctrl_cl = mapa(smem_u32((const void *)sh.ctrl), 0);
    volatile int *ctl = reinterpret_cast<volatile int *>(sh.red + kDLCtlOff);

    int cnt = 0, stop = 0, j0 = 0, batch = 0;
    bool failed = false;
    if (a.debug_flags & 1) {
        // a wait nothing will ever satisfy: exercises the bounded-wait path
        if (!warp_wait<true>(sh.never(), 0u, sh.abort, a.timeout_ns, a.device_status))
            failed = true;
    }
    while (!failed && j0 < N) {
        const int e = batch & 1;
        if (!warp_wait<false>(bars.sums_full + 8u * e, (uint32_t)(batch >> 1) & 1u, sh.abort, a.timeout_ns,
                              a.device_status)) {
            failed = true;
            break;
        }
        const float *red = sh.red + e * (NMF * 34);
        const int nb = reinterpret_cast<const volatile int *>(red)[32];
        if (nb <= 0) {
            failed = true;
            break;
        }
        if constexpr (DET) {
            float tot = 0.f, n0b = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < NMF; ++w2) {
                tot += red[w2 * 34 + (lane & 15)];
                n0b += red[w2 * 34 + 33];
            }
            // statistics and patience exactly as in merge_role, steps 5 and 6
            const float Dp = tot;
            const float Ep = __shfl_down_sync(0xffffffffu, tot, 1);
            const float t = 2.f * Dp + Ep;
            float pre = t;
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
                const float pr = Dp * i0;
                const float x = r0 + pr;
                const float y2 = fmaxf(fmaf(-pr, pr, Ep), 0.f);
                const float d_dir = x > 0.f ? __fdividef(y2, r1 * (r1 + x)) : fmaf(-x, i1, 1.f);
                stable = (d_scale < eps_m) && (d_dir < eps_d);
            }
            const bool stab_k = __shfl_sync(0xffffffffu, stable, 2 * (lane & 7)) && (j0 + (lane & 7) >= 1);
            const uint32_t sbits = __ballot_sync(0xffffffffu, lane < nb && stab_k);
            const int kq = lane & 7;
            const uint32_t zeros = ~sbits & ((2u << kq) - 1u);
            const int run = zeros == 0u ? cnt + kq + 1 : kq - (31 - __clz(zeros));
            const uint32_t hit = __ballot_sync(0xffffffffu, lane < nb && run >= P && j0 + kq + 1 >= minb);
            const int kstop = hit ? __ffs(hit) - 1 : -1;
            cnt = __shfl_sync(0xffffffffu, run, nb - 1);
            if (kstop >= 0) {
                stop = j0 + kstop + 1;
                if (lane == 0) {
                    ctl[3] = stop;
                    mbar_arrive(bars.dec + 8u * e);
                }
                break;
            }
        }
        j0 += nb;
        ++batch;
        if (lane == 0) {
            // batch decided without a stop: its slots go back to the producers
            if constexpr (GM)
                st_release_gpu_u64(gctrl, ep | (uint32_t)j0);
            else
                st_release_cluster_u32(ctrl_cl, (uint32_t)j0);
            if (j0 >= N)
                ctl[3] = N;  // the walk is over (before the arrive: the fold warps read it after their wait)
            mbar_arrive(bars.dec + 8u * e);
        }
    }
    if (!failed && stop == 0)
        stop = N;
    if (lane == 0) {
        if (failed)
            ctl[3] = kDLFailed;
        if constexpr (GM)
            st_release_gpu_u64(gctrl, ep | kStopBit | (failed ? 0u : (uint32_t)stop));
        else
            st_release_cluster_u32(ctrl_cl, kStopBit | (failed ? 0u : (uint32_t)stop));
        a.stop_block[(int64_t)b * a.stop_sb + (int64_t)h * a.stop_sh] = failed ? -1 : stop;
    }
}

// ---- kernel --------------------------------------------------------------------------

// One cluster of C >= 2 CTAs per unit; rank 0 merges (warp 0 decides, warp 1
// forms the shares, warps 2 .. NMF + 1 fold), ranks 1 .. C-1 fetch and
// compute.  Launched with 32 max(2 + NMF, 1 + NW) threads.
template <typename T, int D, int PAGE, int GMAX, int ENGINE, int NMF, bool DET = true>
__global__ void __launch_bounds__(kMaxThreads, 1)
    art_walk_dl_kernel(const KernelArgs a, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int unit = blockIdx.x / a.C;
    const int b = unit / a.Hkv, h = unit % a.Hkv;
    const int Lseq = a.seq_lens[b];
    const int N = Lseq <= 0 ? 0 : Lseq / PAGE + (Lseq % PAGE != 0);
    const bool bad_len = N > a.max_blocks;
    const bool walk = N > 0 && !bad_len;

    const int S = leader ? 0 : a.S;
    const DLLayout L = make_dl_layout(S, a.R, PAGE, D, (int)sizeof(T), GMAX, leader ? a.R : 0);
    const DLLayout LL = make_dl_layout(0, a.R, PAGE, D, (int)sizeof(T), GMAX, a.R);
    Shared sh;
    sh.L.tile_bytes = L.tile_bytes;
    sh.L.stage_bytes = L.stage_bytes;
    sh.L.slot_bytes = L.slot_bytes;
    sh.L.u_off_floats = L.u_off_floats;
    sh.kv = base + L.kv_off;
    sh.ring = reinterpret_cast<float *>(base + L.ring_off);
    sh.pbuf = reinterpret_cast<float *>(base + L.kv_off);  // unused by the tensor-core engine
    sh.red = reinterpret_cast<float *>(base + L.red_off);
    sh.stage_j = reinterpret_cast<uint32_t *>(base + L.meta_off);
    sh.stage_nv = sh.stage_j + S;
    sh.ctrl = reinterpret_cast<volatile uint32_t *>(base);
    sh.fetched = sh.ctrl + 1;
    sh.abort = sh.ctrl + 2;
    sh.bar_ready = smem_u32(base + 16);
    sh.bar_never = sh.bar_ready + 8u * a.R;
    sh.bar_full_k = smem_u32(base + L.bar_off);
    sh.bar_full_v = sh.bar_full_k + 8u * S;
    sh.bar_empty = sh.bar_full_k + 16u * S;
    DLBars bars;
    bars.sums_full = sh.bar_full_k + 24u * S;
    bars.beta_full = bars.sums_full + 16u;
    bars.beta_empty = bars.sums_full + 32u;
    bars.dec = bars.sums_full + 48u;
    bars.landed = bars.sums_full + 64u;
    sh.ring_leader = smem_u32(base + LL.ring_off);
    sh.ready_leader = sh.bar_ready;
    volatile int *ctl = reinterpret_cast<volatile int *>(sh.red + kDLCtlOff);

    const int W = a.C - 1;
    const int wrank = (int)rank - 1;
    int first_lb = -1, first_pp = -1;
    if (walk && !leader && warp == 0) {
        const int jj = wrank + lane * W;
        if (jj < N)
            first_lb = a.block_order ? __ldg(a.block_order + (int64_t)b * a.bo_sb + jj) : (jj == 0 ? 0 : N - jj);
    }
    EngineFor<T, D, PAGE, GMAX, ENGINE> eng;
    if (walk && !leader && warp >= 1 && warp <= a.NW)
        eng.load_q(a, b, h, lane);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(sh.full_k(s), 1);
            mbar_init(sh.full_v(s), 1);
            mbar_init(sh.empty(s), 1);
        }
        for (int r = 0; r < a.R; ++r)
            mbar_init(sh.ready(r), 1);
        mbar_init(sh.never(), 1);
        for (int e = 0; e < 2; ++e) {
            mbar_init(bars.sums_full + 8u * e, NMF);
            mbar_init(bars.beta_full + 8u * e, 1);
            mbar_init(bars.beta_empty + 8u * e, NMF);
            mbar_init(bars.dec + 8u * e, 1);
        }
        sh.ctrl[0] = 0u;
        sh.ctrl[1] = 0u;
        sh.ctrl[2] = 0u;
        ctl[3] = kDLNone;
        fence_mbar_init_cluster();
    }
    __syncthreads();
    if (walk && !leader && warp == 0 && first_lb >= 0 && first_lb < N)
        first_pp = __ldg(a.page_table + (int64_t)b * a.pt_sb + first_lb);
    cluster_sync();  // remote CTAs may now arrive on the merge CTA's barriers

    if (walk) {
        if (leader) {
            if (warp == 0)
                decide_role_dl<D, GMAX, ENGINE, NMF, DET>(a, sh, b, h, N, bars);
            else if (warp == 1)
                share_role_dl<D, GMAX, ENGINE, NMF>(a, sh, N, bars);
            else if (warp <= NMF + 1)
                fold_role_dl<D, GMAX, ENGINE, NMF, DET>(a, sh, b, h, N, warp - 2, bars);
        } else {
            if (warp == 0)
                producer_role<T, D, PAGE, ENGINE, 1>(a, sh, &tmk, &tmv, b, h, N, Lseq, (uint32_t)wrank, W,
                                                         first_lb, first_pp);
            else if (warp <= a.NW)
                compute_role<T, D, PAGE, GMAX, ENGINE, true>(a, sh, b, h, warp - 1, eng);
        }
    } else if (leader && warp == 1) {
        float *op = a.out + (int64_t)b * a.out_sb;
        for (int i = lane; i < a.G * D; i += 32)
            op[(int64_t)(h * a.G + i / D) * a.out_sh + i % D] = 0.f;
        if (lane == 0) {
            a.stop_block[(int64_t)b * a.stop_sb + (int64_t)h * a.stop_sh] = bad_len ? -1 : 0;
            if (bad_len)
                record_error(a.device_status, kErrBadIndex);
        }
    }
    __syncwarp();
    cluster_sync();  // remote stores into the merge CTA are complete
    if (leader && threadIdx.x == 0 && a.blocks_fetched)
        a.blocks_fetched[unit] = (int32_t)sh.fetched[0];
}

}  // namespace art
