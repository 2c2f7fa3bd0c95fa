// art_walk_gr.cuh -- the ART walk with a dedicated merge CTA reached through a
// workspace in global memory, for few (sequence, kv-head) units.
//
// Method as in art_kernels.cuh ("ART: Attention Run-time Termination for
// Efficient Large Language Model Decoding", gist.science explainer, Technical
// Summary 2.1-2.4).  The merge is the one of art_walk_dl.cuh (share warp,
// fold warps, decision warp one batch behind); what differs is that a unit's
// CTAs form no thread-block cluster, so a unit can be served by more CTAs
// than a cluster may hold (one merge CTA and W fetching CTAs per unit, all of
// them resident at once: the launch is cooperative):
//
//   fetching CTAs   producer and compute warps as in art_walk_kernel; a
//                   finished block state is written into the unit's ring in
//                   the workspace (Rg slots), then its slot's ready tag
//                   (epoch, block + 1) is released; the merged count and the
//                   stop are read from the workspace.
//   merge CTA       the share warp polls the ready tags of a batch and copies
//                   its states into a staging ring in shared memory with bulk
//                   copies, then forms the shares as before; the fold and
//                   decision warps are unchanged, and the decision warp
//                   publishes the merged count (freeing the batch's ring
//                   slots) and the stop in the workspace.
//
// Every workspace word carries the call's epoch in its high half, so words
// left by earlier calls are never taken for this call's.
#pragma once

#include "art_walk_dl.cuh"

namespace art {

// Workspace bytes: per unit the merged count, W fetch counts, Rg ready tags
// (8 bytes each) and Rg block states.
__host__ __device__ inline int64_t gr_workspace_bytes(int units, int W, int Rg, uint32_t slot_bytes)
{
    return (int64_t)units * (8 + 8 * (int64_t)W + 8 * (int64_t)Rg) + (int64_t)units * Rg * slot_bytes + 256;
}

// Share warp of the workspace walk: as share_role_dl, but a batch's states
// are first copied from the workspace into the staging ring (slot j % R).
// The copies run one batch ahead: lanes 0-7 own the blocks of the batch whose
// shares come next, lanes 8-15 those of the batch after it; a lane copies its
// block in as soon as the block's ready tag is there (each copy raising the
// bytes its batch's landed barrier waits for), and lane 0 arrives on that
// barrier once the batch is fully requested.  Copying batch b + 1 while the
// shares of batch b are formed is safe: its slots held batch b + 1 - R / 8,
// which is decided (R / 8 >= 6; batch b's shares wait for the fold warps to
// have read batch b - 2, which they do only once batch b - 4 is decided).
template <int D, int GMAX, int ENGINE, int NMF>
__device__ void share_role_gr(const KernelArgs &a, const Shared &sh, int unit, int N, const DLBars &bars)
{
    using MS = MergeShape<D, GMAX, ENGINE, NMF>;
    constexpr int KB = MS::KB, KH = MS::KH, NH = MS::NH;
    static_assert(KB == 8, "two batches of eight blocks over sixteen lanes");
    const int lane = threadIdx.x & 31;
    const int G = a.G;
    const uint32_t slot_bytes = sh.L.slot_bytes;
    const int slot_floats = (int)(slot_bytes / 4);
    volatile int *ctl = reinterpret_cast<volatile int *>(sh.red + kDLCtlOff);
    const int kl = lane / GMAX, gl = lane % GMAX;
    const unsigned long long ep = (unsigned long long)a.epoch << 32;
    const unsigned long long *gfl = a.g_flags + (int64_t)unit * a.Rg;
    const float *gst = a.g_states + (int64_t)unit * a.Rg * slot_floats;
    const uint32_t ring_u = smem_u32(sh.ring);
    float Mx = -CUDART_INF_F, Lm = 0.f;

    bool issued = false;   // this lane's block (j0 + lane, lane < 16) has been requested
    uint32_t arrived = 0;  // lane 0: bit 0 batch b, bit 1 batch b + 1 fully requested (landed arrive done)
    int s0 = 0;
    for (int j0 = 0, batch = 0; j0 < N; ++batch) {
        const int e = batch & 1;
        float *be = sh.red + kDLSumFloats + e * kDLBetaFloats;
        int quit = 0;  // 1 failure, 2 final decision in
        if (batch >= 2) {
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
        const bool has_next = j0 + KB < N;
        // this lane's block: batch b for lanes 0-7, batch b + 1 for lanes 8-15
        const int jk = j0 + lane;
        const bool mine = lane < 16 && jk < N;
        const int eb = lane < 8 ? e : (e ^ 1);
        const uint32_t lbar = bars.landed + 8u * (uint32_t)eb;
        uint64_t t0 = 0;
        bool landed_b = false;
        for (uint32_t it = 0; !quit; ++it) {
            // once the final decision is in, the remaining states never come:
            // the word is read on every pass (a pass waits on global loads)
            if (__shfl_sync(0xffffffffu, lane == 0 && ctl[3] != kDLNone ? 1 : 0, 0)) {
                quit = 2;
                break;
            }
            if (mine && !issued) {
                const unsigned long long v = ld_acquire_gpu_u64(gfl + jk % a.Rg);
                if (v == (ep | (unsigned long long)(jk + 1))) {
                    fence_proxy_async_global();
                    int sl = s0 + lane;
                    while (sl >= a.R)
                        sl -= a.R;
                    mbar_expect_tx(lbar, slot_bytes);
                    bulk_g2s(ring_u + (uint32_t)sl * slot_bytes, gst + (int64_t)(jk % a.Rg) * slot_floats,
                             slot_bytes, lbar);
                    issued = true;
                }
            }
            const uint32_t req = __ballot_sync(0xffffffffu, issued || !mine);
            __syncwarp();
            if (lane == 0) {
                if (!(arrived & 1u) && (req & 0xffu) == 0xffu) {
                    mbar_arrive(bars.landed + 8u * e);
                    arrived |= 1u;
                }
                if (has_next && !(arrived & 2u) && (req & 0xff00u) == 0xff00u) {
                    mbar_arrive(bars.landed + 8u * (e ^ 1));
                    arrived |= 2u;
                }
            }
            const uint32_t arr = __shfl_sync(0xffffffffu, arrived, 0);
            if ((arr & 1u) && mbar_try_wait(bars.landed + 8u * e, (uint32_t)(batch >> 1) & 1u)) {
                landed_b = true;
                break;
            }
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
            // let every copy already requested land before the walk ends
            __syncwarp();
            if (lane == 0) {
                if (!(arrived & 1u))
                    mbar_arrive(bars.landed + 8u * e);
                if (has_next && !(arrived & 2u))
                    mbar_arrive(bars.landed + 8u * (e ^ 1));
            }
            warp_wait<false>(bars.landed + 8u * e, (uint32_t)(batch >> 1) & 1u, sh.abort, a.timeout_ns,
                             a.device_status, false);
            if (has_next)
                warp_wait<false>(bars.landed + 8u * (e ^ 1), (uint32_t)((batch + 1) >> 1) & 1u, sh.abort,
                                 a.timeout_ns, a.device_status, false);
            if (lane == 0)
                reinterpret_cast<volatile int *>(be)[64] = quit == 1 ? -1 : -2;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bars.beta_full + 8u * e);
            break;
        }
        (void)landed_b;
        int sk = s0 + (lane < KB ? lane : 0);
        sk = sk >= a.R ? sk - a.R : sk;
        if (__any_sync(0xffffffffu, lane < nmax && __float_as_uint(sh.ring[(size_t)sk * slot_floats]) != 0u)) {
            // a flagged state (bad order or page entry upstream): the next
            // batch's copies land before the walk ends
            __syncwarp();
            if (lane == 0 && has_next && !(arrived & 2u))
                mbar_arrive(bars.landed + 8u * (e ^ 1));
            if (has_next)
                warp_wait<false>(bars.landed + 8u * (e ^ 1), (uint32_t)((batch + 1) >> 1) & 1u, sh.abort,
                                 a.timeout_ns, a.device_status, false);
            if (lane == 0)
                reinterpret_cast<volatile int *>(be)[64] = -1;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bars.beta_full + 8u * e);
            break;
        }
        const int nb = nmax;
        // shares of the softmax mass, exactly as in share_role_dl
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
        if constexpr (NH > 1)
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
        // advance: the next batch's requests move to lanes 0-7
        const int nxt = __shfl_sync(0xffffffffu, (int)issued, (lane + 8) & 31);
        issued = lane < 8 ? nxt != 0 : false;
        arrived >>= 1;
        j0 += nb;
        s0 += nb;
        if (s0 >= a.R)
            s0 -= a.R;
    }
}

// One merge CTA and W fetching CTAs per unit, consecutive in the grid (no
// clusters; launched cooperatively, so all are resident at once).
template <typename T, int D, int PAGE, int GMAX, int ENGINE, int NMF, bool DET = true>
__global__ void __launch_bounds__(kMaxThreads, 1)
    art_walk_gr_kernel(const KernelArgs a, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per = 1 + a.W;
    const int unit = blockIdx.x / per, rk = blockIdx.x - unit * per;
    const bool leader = rk == 0;
    const int wrank = rk - 1;
    const int b = unit / a.Hkv, h = unit % a.Hkv;
    const int Lseq = a.seq_lens[b];
    const int N = Lseq <= 0 ? 0 : Lseq / PAGE + (Lseq % PAGE != 0);
    const bool bad_len = N > a.max_blocks;
    const bool walk = N > 0 && !bad_len;

    const int S = leader ? 0 : a.S;
    const DLLayout L = make_dl_layout(S, a.R, PAGE, D, (int)sizeof(T), GMAX, leader ? a.R : 0);
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
    sh.ring_leader = 0u;   // no state goes to shared memory of another CTA
    sh.ready_leader = 0u;
    DLBars bars;
    bars.sums_full = sh.bar_full_k + 24u * S;
    bars.beta_full = bars.sums_full + 16u;
    bars.beta_empty = bars.sums_full + 32u;
    bars.dec = bars.sums_full + 48u;
    bars.landed = bars.sums_full + 64u;
    volatile int *ctl = reinterpret_cast<volatile int *>(sh.red + kDLCtlOff);

    int first_lb = -1, first_pp = -1;
    if (walk && !leader && warp == 0) {
        const int jj = wrank + lane * a.W;
        if (jj < N)
            first_lb = a.block_order ? __ldg(a.block_order + (int64_t)b * a.bo_sb + jj) : (jj == 0 ? 0 : N - jj);
    }
    EngineFor<T, D, PAGE, GMAX, ENGINE, 1> eng;
    if (walk && !leader && warp >= 1 && warp <= a.NW)
        eng.load_q(a, b, h, lane);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(sh.full_k(s), 1);
            mbar_init(sh.full_v(s), 1);
            mbar_init(sh.empty(s), 1);
        }
        mbar_init(sh.never(), 1);
        for (int e = 0; e < 2; ++e) {
            mbar_init(bars.sums_full + 8u * e, NMF);
            mbar_init(bars.beta_full + 8u * e, 1);
            mbar_init(bars.beta_empty + 8u * e, NMF);
            mbar_init(bars.dec + 8u * e, 1);
            mbar_init(bars.landed + 8u * e, 1);
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

    if (walk) {
        if (leader) {
            if (warp == 0)
                decide_role_dl<D, GMAX, ENGINE, NMF, DET, true>(a, sh, b, h, N, bars);
            else if (warp == 1)
                share_role_gr<D, GMAX, ENGINE, NMF>(a, sh, unit, N, bars);
            else if (warp <= NMF + 1)
                fold_role_dl<D, GMAX, ENGINE, NMF, DET>(a, sh, b, h, N, warp - 2, bars);
        } else {
            if (warp == 0)
                producer_role<T, D, PAGE, ENGINE, 2>(a, sh, &tmk, &tmv, b, h, N, Lseq, (uint32_t)wrank, a.W,
                                                      first_lb, first_pp);
            else if (warp <= a.NW)
                compute_role<T, D, PAGE, GMAX, ENGINE, true, 1>(a, sh, b, h, warp - 1, eng);
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
    __syncthreads();
    // the merge CTA adds up the pages its unit's fetching CTAs report
    if (leader && threadIdx.x == 0 && a.blocks_fetched) {
        uint32_t total = 0;
        if (walk) {
            const unsigned long long *done = a.g_done + (int64_t)unit * a.W;
            uint64_t t0 = 0;
            for (int w = 0; w < a.W; ++w) {
                for (uint32_t it = 0;; ++it) {
                    const unsigned long long v = ld_acquire_gpu_u64(done + w);
                    if ((uint32_t)(v >> 32) == a.epoch) {
                        total += (uint32_t)v;
                        break;
                    }
                    if ((it & 15u) == 15u) {
                        const uint64_t now = global_timer_ns();
                        if (t0 == 0)
                            t0 = now;
                        if ((int64_t)(now - t0) > a.timeout_ns) {
                            record_error(a.device_status, kErrTimeout);
                            break;
                        }
                    }
                }
            }
        }
        a.blocks_fetched[unit] = (int32_t)total;
    }
}

}  // namespace art
