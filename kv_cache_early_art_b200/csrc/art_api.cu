// art_api.cu -- host side of libart: argument checks, TMA descriptors, launch
// shape selection and the extern "C" entry points declared in include/art.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <atomic>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <unordered_map>

#include "../../include/art.h"
#include "art_host.h"
#include "art_kernels.cuh"
#include "art_walk.h"
#include "art_walk_dl.cuh"
#include "art_walk_gr.cuh"

namespace {

using art::KernelArgs;

// Default walk order: [0, N-1, N-2, ..., 1], -1 beyond N.
__global__ void art_build_order_kernel(const int32_t *seq_lens, int B, int page, int32_t *order, int64_t row_stride,
                                       int max_blocks)
{
    const int b = blockIdx.y;
    if (b >= B)
        return;
    const int L = seq_lens[b];
    const int N = L <= 0 ? 0 : L / page + (L % page != 0);
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < max_blocks; j += gridDim.x * blockDim.x)
        order[(int64_t)b * row_stride + j] = j < N ? (j == 0 ? 0 : N - j) : -1;
}

using art::Layout;

// ---------------------------------------------------------------- checks ----

using art_host::aligned;
using art_host::elem_size;
using art_host::is_null;

struct Problem {
    int dtype;
    int B, Hq, Hkv, G, d, page, max_blocks, num_pages;
    // query tokens sharing one walk; G = NQ * GQ rows per unit
    int NQ = 1, GQ = 0;
    int64_t q_st = 0, out_st = 0, stop_st = 0;
};

art_status_t check_tensors(const art_params_t *p, Problem *pr)
{
    const art_tensor_t *q = &p->q, *k = &p->k_cache, *v = &p->v_cache, *pt = &p->page_table,
                       *bo = &p->block_order, *sl = &p->seq_lens, *o = &p->out, *st = &p->stop_block;
    // block_order may be absent (NULL data): the default order is then built on the fly
    const bool has_order = bo->data != nullptr;
    if (is_null(q) || is_null(k) || is_null(v) || is_null(pt) || is_null(sl) || is_null(o) || is_null(st))
        return ART_ERR_NULL;
    if (q->ndim != 3 || k->ndim != 4 || v->ndim != 4 || pt->ndim != 2 || (has_order && bo->ndim != 2) ||
        sl->ndim != 1 || o->ndim != 3 || st->ndim != 2)
        return ART_ERR_SHAPE;
    if (q->dtype != ART_F32 && q->dtype != ART_BF16)
        return ART_ERR_DTYPE;
    if (k->dtype != q->dtype || v->dtype != q->dtype || pt->dtype != ART_I32 || (has_order && bo->dtype != ART_I32) ||
        sl->dtype != ART_I32 || o->dtype != ART_F32 || st->dtype != ART_I32)
        return ART_ERR_DTYPE;
    const int64_t B = q->shape[0], Hq = q->shape[1], d = q->shape[2];
    const int64_t NP = k->shape[0], Hkv = k->shape[1], page = k->shape[2];
    if (B <= 0 || Hq <= 0 || d <= 0 || NP <= 0 || Hkv <= 0 || page <= 0)
        return ART_ERR_SHAPE;
    if (B > (1 << 24) || Hq > 4096 || NP > (int64_t)INT32_MAX || Hkv > 4096)
        return ART_ERR_SHAPE;
    for (int i = 0; i < 4; ++i)
        if (v->shape[i] != k->shape[i])
            return ART_ERR_SHAPE;
    if (k->shape[3] != d || Hq % Hkv != 0)
        return ART_ERR_SHAPE;
    if (pt->shape[0] != B || (has_order && (bo->shape[0] != B || pt->shape[1] != bo->shape[1])) ||
        pt->shape[1] <= 0 || pt->shape[1] > (int64_t)INT32_MAX / 256 || sl->shape[0] != B)
        return ART_ERR_SHAPE;
    if (o->shape[0] != B || o->shape[1] != Hq || o->shape[2] != d || st->shape[0] != B || st->shape[1] != Hkv)
        return ART_ERR_SHAPE;
    // contiguity and alignment the kernels rely on
    const int64_t es = elem_size(q->dtype);
    if (q->stride[2] != 1 || k->stride[3] != 1 || v->stride[3] != 1 || pt->stride[1] != 1 ||
        (has_order && bo->stride[1] != 1) || sl->stride[0] != 1 || o->stride[2] != 1)
        return ART_ERR_SHAPE;
    if (!aligned(q->data, 16) || (q->stride[0] * es) % 16 || (q->stride[1] * es) % 16 || q->stride[0] < 0 ||
        q->stride[1] < 0)
        return ART_ERR_SHAPE;
    for (const art_tensor_t *c : {k, v}) {
        if (!aligned(c->data, 16))
            return ART_ERR_SHAPE;
        for (int i = 0; i < 3; ++i)
            if (c->stride[i] <= 0 || (c->stride[i] * es) % 16 || c->stride[i] * es >= (int64_t)1 << 40)
                return ART_ERR_SHAPE;
    }
    if (!aligned(pt->data, 4) || (has_order && !aligned(bo->data, 4)) || !aligned(sl->data, 4) || !aligned(o->data, 4) ||
        !aligned(st->data, 4))
        return ART_ERR_SHAPE;
    const int64_t G = Hq / Hkv;
    if (!(d == 64 || d == 128) || !(page == 16 || page == 64) || G > 8)
        return ART_ERR_UNSUPPORTED;
    pr->dtype = q->dtype;
    pr->B = (int)B;
    pr->Hq = (int)Hq;
    pr->Hkv = (int)Hkv;
    pr->G = (int)G;
    pr->d = (int)d;
    pr->page = (int)page;
    pr->max_blocks = (int)pt->shape[1];
    pr->num_pages = (int)NP;
    if ((int64_t)B * Hkv > (int64_t)INT32_MAX / 16)
        return ART_ERR_SHAPE;
    return ART_OK;
}

// Several query tokens per sequence: q and out are [B, T, Hq, d], stop_block
// [B, T, Hkv].  Token 0's slices go through the single-query checks; the
// token dimension is checked here.
art_status_t check_tensors_multi(const art_params_t *p, int nq, Problem *pr)
{
    const art_tensor_t *q = &p->q, *o = &p->out, *st = &p->stop_block;
    if (is_null(q) || is_null(o) || is_null(st))
        return ART_ERR_NULL;
    if (q->ndim != 4 || o->ndim != 4 || st->ndim != 3)
        return ART_ERR_SHAPE;
    if (q->shape[1] != nq || o->shape[1] != nq || st->shape[1] != nq)
        return ART_ERR_SHAPE;
    art_params_t v = *p;
    auto drop_token_dim = [](const art_tensor_t &t, art_tensor_t *r) {
        *r = t;
        r->ndim = t.ndim - 1;
        r->shape[0] = t.shape[0];
        r->stride[0] = t.stride[0];
        for (int i = 1; i < r->ndim; ++i) {
            r->shape[i] = t.shape[i + 1];
            r->stride[i] = t.stride[i + 1];
        }
        for (int i = r->ndim; i < 4; ++i) {
            r->shape[i] = 0;
            r->stride[i] = 0;
        }
    };
    drop_token_dim(*q, &v.q);
    drop_token_dim(*o, &v.out);
    drop_token_dim(*st, &v.stop_block);
    art_status_t s = check_tensors(&v, pr);
    if (s != ART_OK)
        return s;
    const int64_t es = elem_size(q->dtype);
    if (q->stride[1] < 0 || (q->stride[1] * es) % 16 || o->stride[1] < 0 || st->stride[1] < 0)
        return ART_ERR_SHAPE;
    if (nq > 1 && ((int64_t)nq * pr->G > 8 || pr->d != 128))
        return ART_ERR_UNSUPPORTED;  // every token's heads must fit one unit's eight rows
    pr->NQ = nq;
    pr->GQ = pr->G;
    pr->G = nq * pr->G;
    pr->q_st = q->stride[1];
    pr->out_st = o->stride[1];
    pr->stop_st = st->stride[1];
    return ART_OK;
}

art_status_t check_params(const art_params_t *p)
{
    if (std::isnan(p->eps_m) || std::isnan(p->eps_d) || p->eps_m < 0.f || p->eps_d < 0.f || p->P < 0 ||
        p->min_blocks < 0)
        return ART_ERR_PARAM;
    if (std::isnan(p->sm_scale) || std::isinf(p->sm_scale))
        return ART_ERR_PARAM;
    if (p->engine < 0 || p->engine > 2 || p->cluster_size < 0 || p->cluster_size > 16 || p->stages < 0 ||
        p->stages > 8 || p->compute_warps < 0 || p->compute_warps > art::kMaxComputeWarps || p->window < 0 ||
        p->window > 128 || p->timeout_ns < 0 || (p->debug_flags & ~1) || p->prefetch < -1 || p->prefetch > 64 ||
        p->detector_off < 0 || p->detector_off > 1 || p->merge_cta < -1 || p->merge_cta > 2 ||
        p->workspace_bytes < 0)
        return ART_ERR_PARAM;
    if (p->stages == 1 || (p->window > 0 && p->window < art::kMinWindow))
        return ART_ERR_PARAM;
    if (p->workspace && !aligned(p->workspace, 256))
        return ART_ERR_SHAPE;
    for (const void *ptr : {(const void *)p->eps_m_per_seq, (const void *)p->eps_d_per_seq,
                            (const void *)p->P_per_seq, (const void *)p->min_blocks_per_seq,
                            (const void *)p->blocks_fetched, (const void *)p->device_status})
        if (ptr && !aligned(ptr, 4))
            return ART_ERR_SHAPE;
    return ART_OK;
}

// ------------------------------------------------------------- kernels ----

using art_walk::KernelFn;

template <int ENGINE, int GMAX, int NMW>
int merge_warps_dg(int d)
{
    return d == 64 ? art::MergeShape<64, GMAX, ENGINE, NMW>::NM : art::MergeShape<128, GMAX, ENGINE, NMW>::NM;
}

// Warps the kernel instantiation devotes to the merge (compile-time in the
// kernel).  Four merge warps shorten the per-unit merge when units are few;
// one keeps CTAs small enough for two per SM when units are many.  The
// CUDA-core engine always uses one.
int merge_warps(int engine, int d, int gmax, int nmw)
{
    if (engine == art::kEngineMma) {
        if (nmw == 4)
            return gmax == 4 ? merge_warps_dg<art::kEngineMma, 4, 4>(d) : merge_warps_dg<art::kEngineMma, 8, 4>(d);
        return gmax == 4 ? merge_warps_dg<art::kEngineMma, 4, 1>(d) : merge_warps_dg<art::kEngineMma, 8, 1>(d);
    }
    if (gmax == 1)
        return merge_warps_dg<art::kEngineCuda, 1, 1>(d);
    return gmax == 4 ? merge_warps_dg<art::kEngineCuda, 4, 1>(d) : merge_warps_dg<art::kEngineCuda, 8, 1>(d);
}

int gmax_for(int G, int engine)
{
    if (engine == art::kEngineMma)
        return G <= 4 ? 4 : 8;
    return G <= 1 ? 1 : (G <= 4 ? 4 : 8);
}

KernelFn pick_kernel(int dtype, int engine, int d, int page, int gmax, int nmw, bool detector)
{
    if (dtype == ART_F32)
        return art_walk::f32_cuda(gmax, d, page, detector);
    if (engine == art::kEngineMma)
        return art_walk::bf16_mma(gmax, nmw, d, page, detector);
    return detector ? art_walk::bf16_cuda(gmax, d, page) : nullptr;
}

KernelFn pick_kernel_multi(int dtype, int engine, int page, int gmax, int nmw)
{
    return art_walk::multi(dtype == ART_F32, engine, page, gmax, nmw);
}

// ------------------------------------------------------ device caches ----

struct DeviceInfo {
    int sms = 0, smem_optin = 0, smem_sm = 0, smem_reserved = 0;
};

std::mutex g_mu;
std::unordered_map<int, DeviceInfo> g_dev;
std::unordered_map<const void *, int> g_smem_set;   // kernel -> dynamic smem limit already set

art_status_t device_info(DeviceInfo *out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return ART_ERR_LAUNCH;
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_dev.find(dev);
    if (it == g_dev.end()) {
        DeviceInfo di;
        if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&di.smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&di.smem_reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
            return ART_ERR_LAUNCH;
        it = g_dev.emplace(dev, di).first;
    }
    *out = it->second;
    return ART_OK;
}

art_status_t prepare_kernel(KernelFn fn, int smem)
{
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_smem_set.find((const void *)fn);
    if (it != g_smem_set.end() && it->second >= smem)
        return ART_OK;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
        cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return ART_ERR_LAUNCH;
    g_smem_set[(const void *)fn] = smem;
    return ART_OK;
}

// ---------------------------------------------------------- tensor maps ----

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 4-D view [num_pages, Hkv, page, d] of a cache; box = one page of one head
// (d columns, or 64-column slabs with the 128-byte swizzle for the MMA engine).
art_status_t make_cache_map(CUtensorMap *map, const art_tensor_t *c, int dtype, bool swizzle)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return ART_ERR_LAUNCH;
    const int64_t es = elem_size(dtype);
    cuuint64_t dims[4] = {(cuuint64_t)c->shape[3], (cuuint64_t)c->shape[2], (cuuint64_t)c->shape[1],
                          (cuuint64_t)c->shape[0]};
    cuuint64_t strides[3] = {(cuuint64_t)(c->stride[2] * es), (cuuint64_t)(c->stride[1] * es),
                             (cuuint64_t)(c->stride[0] * es)};
    cuuint32_t box[4] = {(cuuint32_t)(swizzle ? 64 : c->shape[3]), (cuuint32_t)c->shape[2], 1u, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUresult r = enc(map, dtype == ART_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                           4, c->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ART_OK : ART_ERR_LAUNCH;
}

// -------------------------------------------------------------- launch ----

struct Shape {
    int engine, gmax, nmw, S, NW, R, C, PF, smem, threads;
    int RF = 0;              // window (blocks fetched ahead of the merged prefix); R = ring slots
    int dl = 0;              // 1: dedicated merge CTA (art_walk_dl_kernel); 2: through the workspace
    int W = 0, Rg = 0;       // workspace walk: fetching CTAs per unit, ring slots per unit
    KernelFn fn = nullptr;   // set by the dedicated-merge choice
};

// clusters of C CTAs of fn (threads, smem) that can be resident at once (0 if none)
int resident_clusters(KernelFn fn, int threads, int smem, int units, int C)
{
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(units * C);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, (void *)fn, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return nclusters;
}

int smem_bytes(const Shape &s, const Problem &pr)
{
    const Layout L = art::make_layout(s.S, s.NW, s.R, pr.page, pr.d, (int)elem_size(pr.dtype), s.gmax,
                                      s.engine != art::kEngineMma);
    return (int)L.total + 1024;  // slack to align the base to 1024 bytes
}

art_status_t choose_shape(const art_params_t *p, const Problem &pr, const DeviceInfo &di, Shape *out)
{
    Shape s;
    s.engine = p->engine ? p->engine : (pr.dtype == ART_BF16 ? art::kEngineMma : art::kEngineCuda);
    if (s.engine == art::kEngineMma && pr.dtype != ART_BF16)
        return ART_ERR_UNSUPPORTED;
    s.gmax = gmax_for(pr.G, s.engine);
    s.C = p->cluster_size;
    s.nmw = (s.engine == art::kEngineMma && pr.B * pr.Hkv < di.sms) ? 4 : 1;
    const int tile = pr.page * pr.d * (int)elem_size(pr.dtype);
    const int units = pr.B * pr.Hkv;
    // L2 prefetch ahead of the staged loads: off unless asked for (measured on
    // the B200 it does not shorten the walk and it costs L2 space at high batch)
    s.PF = p->prefetch > 0 ? p->prefetch : 0;
    // (compute warps, stages, window) in order of preference.  With at least
    // one unit per SM, two small CTAs per SM keep the most pages in flight;
    // with fewer units each unit is split over a cluster and needs a deeper
    // window to cover the latency from fetch to merged stop decision.
    static const int many_units[][3] = {{2, 2, 16}, {1, 2, 16}, {2, 2, 8}, {1, 2, 8}};
    // many units whose state ring is too large for two CTAs per SM (eight
    // rows per unit): one CTA per SM with the same pages in flight
    static const int many_units_wide[][3] = {{4, 4, 16}, {3, 3, 16}, {2, 2, 16}, {1, 2, 8}};
    static const int few_units_large[][3] = {{5, 5, 28}, {4, 4, 24}, {2, 4, 24}, {3, 3, 24}, {2, 2, 24},
                                             {2, 4, 16}, {2, 2, 16}, {1, 2, 16}, {1, 2, 8}};
    static const int few_units_small[][3] = {{4, 8, 32}, {4, 8, 16}, {4, 4, 16}, {2, 4, 16}, {2, 2, 8},
                                             {1, 2, 8}};
    const int(*cand)[3];
    int ncand;
    if (units >= di.sms) {
        cand = many_units;
        ncand = 4;
        Shape t = s;
        t.NW = t.S = 2;
        t.R = 16;
        if (2 * (smem_bytes(t, pr) + di.smem_reserved) > di.smem_sm)
            cand = many_units_wide;
    } else if (tile >= 16384) {
        cand = few_units_large;
        ncand = 9;
    } else {
        cand = few_units_small;
        ncand = 6;
    }
    // every compute warp owns the same stages (stage i goes to warp i % NW),
    // so S must be a multiple of NW: only a caller who fixes both can break that
    if (p->compute_warps && p->stages && p->stages % p->compute_warps != 0)
        return ART_ERR_PARAM;
    for (int i = 0; i < ncand; ++i) {
        int NW = p->compute_warps ? p->compute_warps : cand[i][0];
        int S = p->stages ? p->stages : cand[i][1];
        if (p->stages && !p->compute_warps) {
            // stages fixed, warps automatic: the largest warp count up to the
            // candidate's that divides the stages
            while (S % NW != 0)
                --NW;
        } else if (!p->stages) {
            // warps fixed (or both automatic): round the candidate's stages up
            // to a multiple of the warps, and down again past the 8-stage limit
            S = NW * ((S + NW - 1) / NW);
            if (S > 8)
                S = NW * (8 / NW);
        }
        s.NW = NW;
        s.S = S;
        s.R = p->window ? p->window : cand[i][2];
        s.RF = s.R;
        s.threads = 32 * (1 + merge_warps(s.engine, pr.d, s.gmax, s.nmw) + NW);
        s.smem = smem_bytes(s, pr);
        if (s.smem <= di.smem_optin) {
            *out = s;
            return ART_OK;
        }
        if (p->compute_warps && p->stages && p->window)
            break;
    }
    return ART_ERR_UNSUPPORTED;
}

art_status_t pick_cluster(KernelFn fn, Shape *s, const Problem &pr, const DeviceInfo &di, KernelArgs &ka)
{
    const int units = pr.B * pr.Hkv;
    if (s->C > 0)
        return ART_OK;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, s->threads, s->smem) != cudaSuccess)
        return ART_ERR_LAUNCH;
    per_sm = per_sm < 1 ? 1 : per_sm;
    const int slots = di.sms * per_sm;
    auto resident = [&](int C) -> int { return resident_clusters(fn, s->threads, s->smem, units, C); };
    int C = 1;
    if (units < slots) {
        // one wave: the largest cluster size whose clusters all fit at once
        C = slots / units;
        C = C > 16 ? 16 : C;
        for (; C > 1; --C)
            if (resident(C) >= units)
                break;
    } else {
        // several waves of units: a unit split over C CTAs takes about 1/C of
        // the time, and the launch takes ceil(units / resident clusters)
        // rounds, so pick the C with the fewest rounds / C (the smaller C on
        // a tie: it has no cross-CTA merge traffic)
        long best_num = (units + slots - 1) / slots, best_den = 1;   // C = 1
        for (int c = 2; c <= 4; c *= 2) {
            const int rc = resident(c);
            if (rc <= 0)
                continue;
            const long rounds = (units + rc - 1) / rc;
            if (rounds * best_den < best_num * c) {
                best_num = rounds;
                best_den = c;
                C = c;
            }
        }
    }
    s->C = C;
    (void)ka;
    return ART_OK;
}

// Dedicated merge CTA (art_walk_dl_kernel): rank 0 of each cluster holds the
// state ring in all of its shared memory and only merges; the other ranks
// fetch and compute.  Chosen automatically for fewer units than SMs when at
// least four CTAs per unit fit at once (the merge CTA costs one fetching CTA,
// so small clusters keep art_walk_kernel); merge_cta = 1 asks for it.
// *chosen stays false when art_walk_kernel should run instead.
art_status_t choose_dl(const art_params_t *p, const Problem &pr, const DeviceInfo &di, Shape *out, bool *chosen)
{
    *chosen = false;
    const bool forced = p->merge_cta == 1;
    const int engine = p->engine ? p->engine : (pr.dtype == ART_BF16 ? art::kEngineMma : art::kEngineCuda);
    if (engine != art::kEngineMma || pr.dtype != ART_BF16 || pr.d != 128 || pr.page != 64)
        return forced ? ART_ERR_UNSUPPORTED : ART_OK;
    const int units = pr.B * pr.Hkv;
    if (!forced && units >= di.sms)
        return ART_OK;
    if (p->cluster_size == 1)
        return forced ? ART_ERR_PARAM : ART_OK;
    if (p->compute_warps && p->stages && p->stages % p->compute_warps != 0)
        return ART_ERR_PARAM;
    Shape s;
    s.engine = art::kEngineMma;
    s.gmax = gmax_for(pr.G, s.engine);
    s.nmw = s.gmax;  // one fold warp per 16 output floats of a lane: 4 or 8
    s.PF = p->prefetch > 0 ? p->prefetch : 0;
    s.dl = 1;
    const int es = (int)elem_size(pr.dtype);
    const int limit = di.smem_optin - 1024;  // slack to align the base to 1024 bytes
    // the merge CTA's ring: as deep as fits, in whole merge batches, at most
    // 64 slots and at most the window
    const int cap = p->window && p->window < 64 ? p->window : 64;
    int R = cap;
    for (; R > art::kMinWindow; R -= R % 8 ? R % 8 : 8)
        if ((int)art::make_dl_layout(0, R, pr.page, pr.d, es, s.gmax, R).total <= limit)
            break;
    if ((int)art::make_dl_layout(0, R, pr.page, pr.d, es, s.gmax, R).total > limit)
        return forced ? ART_ERR_UNSUPPORTED : ART_OK;
    s.R = R;
    // the fetching CTAs: (compute warps, stages), deepest first
    static const int cand[][2] = {{6, 6}, {3, 6}, {5, 5}, {4, 4}, {2, 4}, {2, 2}, {1, 2}};
    bool fit = false;
    for (const auto &c : cand) {
        int NW = p->compute_warps ? p->compute_warps : c[0];
        int S = p->stages ? p->stages : c[1];
        if (p->stages && !p->compute_warps) {
            while (S % NW != 0)
                --NW;
        } else if (!p->stages) {
            S = NW * ((S + NW - 1) / NW);
            if (S > 8)
                S = NW * (8 / NW);
        }
        if ((int)art::make_dl_layout(S, R, pr.page, pr.d, es, s.gmax, 0).total <= limit) {
            s.NW = NW;
            s.S = S;
            fit = true;
            break;
        }
    }
    if (!fit)
        return forced ? ART_ERR_UNSUPPORTED : ART_OK;
    const int lead = (int)art::make_dl_layout(0, R, pr.page, pr.d, es, s.gmax, R).total;
    const int work = (int)art::make_dl_layout(s.S, R, pr.page, pr.d, es, s.gmax, 0).total;
    s.smem = (lead > work ? lead : work) + 1024;
    s.threads = 32 * (2 + s.nmw > 1 + s.NW ? 2 + s.nmw : 1 + s.NW);
    s.fn = art_walk::bf16_mma_dl(s.gmax, pr.d, pr.page, !p->detector_off);
    if (!s.fn)
        return forced ? ART_ERR_UNSUPPORTED : ART_OK;
    art_status_t st = prepare_kernel(s.fn, s.smem);
    if (st != ART_OK)
        return st;
    int C = p->cluster_size;
    if (!C) {
        // the largest cluster whose clusters are all resident at once
        C = di.sms / units;
        C = C > 16 ? 16 : C;
        for (; C > 2; --C)
            if (resident_clusters(s.fn, s.threads, s.smem, units, C) >= units)
                break;
        if (C < 2 || resident_clusters(s.fn, s.threads, s.smem, units, C) < 1)
            return forced ? ART_ERR_UNSUPPORTED : ART_OK;
        if (!forced && C < 4)
            return ART_OK;
    }
    s.C = C;
    // the window reaches past the ring by two merge batches (at most the pages
    // the fetching CTAs can hold in their stages): those are fetched and
    // computed while the merge still holds every slot, and their states wait
    // for a slot (slot_gate).  A deeper window read more pages past the stop
    // on the few-unit workloads without a faster walk.
    const int past = (C - 1) * s.S < 16 ? (C - 1) * s.S : 16;
    s.RF = p->window ? p->window : s.R + past;
    s.RF = s.RF > 128 ? 128 : s.RF;
    if (s.RF < s.R)
        s.RF = s.R;
    *out = s;
    *chosen = true;
    return ART_OK;
}

// The dedicated merge reached through a workspace (art_walk_gr_kernel), on
// request (merge_cta = 2): one merge CTA and W fetching CTAs per unit, as many
// as fit on the GPU at once (the launch is cooperative).  need: the workspace
// this problem can use (a ring of 128 slots per unit), also when none is
// given.  *chosen stays false when another walk should run instead.
art_status_t choose_gr(const art_params_t *p, const Problem &pr, const DeviceInfo &di, Shape *out, bool *chosen,
                       int64_t *need)
{
    *chosen = false;
    *need = 0;
    const bool forced = p->merge_cta == 2;
    const int engine = p->engine ? p->engine : (pr.dtype == ART_BF16 ? art::kEngineMma : art::kEngineCuda);
    if (engine != art::kEngineMma || pr.dtype != ART_BF16 || pr.d != 128 || pr.page != 64)
        return forced ? ART_ERR_UNSUPPORTED : ART_OK;
    const int units = pr.B * pr.Hkv;
    if (!forced && units >= di.sms)
        return ART_OK;
    if (p->compute_warps && p->stages && p->stages % p->compute_warps != 0)
        return ART_ERR_PARAM;
    Shape s;
    s.engine = art::kEngineMma;
    s.gmax = gmax_for(pr.G, s.engine);
    s.nmw = s.gmax;
    s.PF = p->prefetch > 0 ? p->prefetch : 0;
    s.dl = 2;
    const int es = (int)elem_size(pr.dtype);
    const int limit = di.smem_optin - 1024;
    // the merge CTA's staging ring: at least five merge batches deep (a batch
    // is copied in only once the batch five before it has been decided)
    int R = 64;
    for (; R > 40; R -= 8)
        if ((int)art::make_dl_layout(0, R, pr.page, pr.d, es, s.gmax, R).total <= limit)
            break;
    if ((int)art::make_dl_layout(0, R, pr.page, pr.d, es, s.gmax, R).total > limit)
        return forced ? ART_ERR_UNSUPPORTED : ART_OK;
    s.R = R;
    static const int cand[][2] = {{6, 6}, {3, 6}, {5, 5}, {4, 4}, {2, 4}, {2, 2}, {1, 2}};
    bool fit = false;
    for (const auto &c : cand) {
        int NW = p->compute_warps ? p->compute_warps : c[0];
        int S = p->stages ? p->stages : c[1];
        if (p->stages && !p->compute_warps) {
            while (S % NW != 0)
                --NW;
        } else if (!p->stages) {
            S = NW * ((S + NW - 1) / NW);
            if (S > 8)
                S = NW * (8 / NW);
        }
        if ((int)art::make_dl_layout(S, R, pr.page, pr.d, es, s.gmax, 0).total <= limit) {
            s.NW = NW;
            s.S = S;
            fit = true;
            break;
        }
    }
    if (!fit)
        return forced ? ART_ERR_UNSUPPORTED : ART_OK;
    const int lead = (int)art::make_dl_layout(0, R, pr.page, pr.d, es, s.gmax, R).total;
    const int work = (int)art::make_dl_layout(s.S, R, pr.page, pr.d, es, s.gmax, 0).total;
    s.smem = (lead > work ? lead : work) + 1024;
    s.threads = 32 * (2 + s.nmw > 1 + s.NW ? 2 + s.nmw : 1 + s.NW);
    s.fn = art_walk::bf16_mma_gr(s.gmax, pr.d, pr.page, !p->detector_off);
    if (!s.fn)
        return forced ? ART_ERR_UNSUPPORTED : ART_OK;
    art_status_t st = prepare_kernel(s.fn, s.smem);
    if (st != ART_OK)
        return st;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, s.fn, s.threads, s.smem) != cudaSuccess) {
        cudaGetLastError();
        return ART_ERR_LAUNCH;
    }
    const int slots = di.sms * (per_sm < 1 ? 0 : per_sm);
    const int W = p->cluster_size ? p->cluster_size - 1 : (slots / units) - 1;
    if (W < (forced ? 1 : 3) || (int64_t)units * (1 + W) > slots)
        return forced ? ART_ERR_UNSUPPORTED : ART_OK;
    s.W = W;
    s.C = 1 + W;
    const uint32_t slot = art::make_dl_layout(0, R, pr.page, pr.d, es, s.gmax, R).slot_bytes;
    *need = art::gr_workspace_bytes(units, W, 128, slot);
    if (!p->workspace)
        return forced ? ART_ERR_NULL : ART_OK;
    int Rg = 128;
    while (Rg > 16 && art::gr_workspace_bytes(units, W, Rg, slot) > p->workspace_bytes)
        Rg -= 8;
    if (art::gr_workspace_bytes(units, W, Rg, slot) > p->workspace_bytes)
        return forced ? ART_ERR_SHAPE : ART_OK;
    s.Rg = Rg;
    // the window: blocks fetched ahead of the merged count, within the ring
    s.RF = p->window ? (p->window < Rg ? p->window : Rg) : Rg;
    *out = s;
    *chosen = true;
    return ART_OK;
}

std::atomic<uint32_t> g_epoch{0};

// tokens_dim: q and out are [B, T, Hq, d] and stop_block [B, T, Hkv] (T = nq)
art_status_t launch(const art_params_t *p, art_stream_t stream, int nq = 1, bool tokens_dim = false)
{
    Problem pr;
    art_status_t st = tokens_dim ? check_tensors_multi(p, nq, &pr) : check_tensors(p, &pr);
    if (st != ART_OK)
        return st;
    st = check_params(p);
    if (st != ART_OK)
        return st;
    if (p->engine == art::kEngineMma && pr.dtype != ART_BF16)
        return ART_ERR_UNSUPPORTED;

    DeviceInfo di;
    if ((st = device_info(&di)) != ART_OK)
        return st;
    if (nq > 1 && p->detector_off)
        return ART_ERR_UNSUPPORTED;
    if (nq > 1 && p->merge_cta == 1)
        return ART_ERR_UNSUPPORTED;
    if (nq > 1 && p->merge_cta == 2)
        return ART_ERR_UNSUPPORTED;
    Shape s;
    bool dl = false, gr = false;
    if (nq == 1 && p->merge_cta == 2) {
        int64_t need = 0;
        if ((st = choose_gr(p, pr, di, &s, &gr, &need)) != ART_OK)
            return st;
    }
    if (!gr && nq == 1 && p->merge_cta != -1 && p->merge_cta != 2 && (st = choose_dl(p, pr, di, &s, &dl)) != ART_OK)
        return st;
    KernelFn fn = nullptr;
    if (dl || gr) {
        fn = s.fn;
    } else {
        if ((st = choose_shape(p, pr, di, &s)) != ART_OK)
            return st;
        fn = nq > 1 ? pick_kernel_multi(pr.dtype, s.engine, pr.page, s.gmax, s.nmw)
                    : pick_kernel(pr.dtype, s.engine, pr.d, pr.page, s.gmax, s.nmw, !p->detector_off);
        if (!fn)
            return ART_ERR_UNSUPPORTED;
        if ((st = prepare_kernel(fn, s.smem)) != ART_OK)
            return st;
    }

    KernelArgs ka;
    std::memset(&ka, 0, sizeof ka);
    // with several tokens the head stride is the one after the token dimension
    const int hd = tokens_dim ? 2 : 1;
    ka.q = p->q.data;
    ka.q_sb = p->q.stride[0];
    ka.q_sh = p->q.stride[hd];
    ka.out = static_cast<float *>(p->out.data);
    ka.out_sb = p->out.stride[0];
    ka.out_sh = p->out.stride[hd];
    ka.stop_block = static_cast<int32_t *>(p->stop_block.data);
    ka.stop_sb = p->stop_block.stride[0];
    ka.stop_sh = p->stop_block.stride[hd];
    ka.page_table = static_cast<const int32_t *>(p->page_table.data);
    ka.pt_sb = p->page_table.stride[0];
    ka.block_order = static_cast<const int32_t *>(p->block_order.data);
    ka.bo_sb = p->block_order.stride[0];
    ka.seq_lens = static_cast<const int32_t *>(p->seq_lens.data);
    ka.eps_m_arr = p->eps_m_per_seq;
    ka.eps_d_arr = p->eps_d_per_seq;
    ka.P_arr = p->P_per_seq;
    ka.minb_arr = p->min_blocks_per_seq;
    ka.eps_m = p->eps_m;
    ka.eps_d = p->eps_d;
    ka.P = p->P;
    ka.min_blocks = p->min_blocks;
    const float scale = p->sm_scale > 0.f ? p->sm_scale : 1.0f / std::sqrt((float)pr.d);
    ka.scale_log2 = scale * 1.4426950408889634f;
    ka.blocks_fetched = p->blocks_fetched;
    ka.device_status = p->device_status;
    ka.B = pr.B;
    ka.Hq = pr.Hq;
    ka.Hkv = pr.Hkv;
    ka.G = pr.G;
    ka.num_pages = pr.num_pages;
    ka.max_blocks = pr.max_blocks;
    ka.timeout_ns = p->timeout_ns > 0 ? p->timeout_ns : 2000000000LL;
    ka.debug_flags = p->debug_flags;
    ka.NQ = pr.NQ;
    ka.GQ = nq == 1 ? pr.G : pr.GQ;
    ka.q_st = pr.q_st;
    ka.out_st = pr.out_st;
    ka.stop_st = pr.stop_st;

    if (!dl && !gr && (st = pick_cluster(fn, &s, pr, di, ka)) != ART_OK)
        return st;
    ka.C = s.C;
    ka.S = s.S;
    ka.NW = s.NW;
    ka.R = s.R;
    ka.RF = s.RF;
    if (gr) {
        // the workspace: merged counts, fetch counts, ready tags, states
        const int units = pr.B * pr.Hkv;
        uint8_t *ws = static_cast<uint8_t *>(p->workspace);
        ka.g_ctrl = reinterpret_cast<unsigned long long *>(ws);
        ka.g_done = ka.g_ctrl + units;
        ka.g_flags = ka.g_done + (int64_t)units * s.W;
        const uintptr_t st0 = reinterpret_cast<uintptr_t>(ka.g_flags + (int64_t)units * s.Rg);
        ka.g_states = reinterpret_cast<float *>((st0 + 255) & ~(uintptr_t)255);
        uint32_t e = ++g_epoch;
        if (e == 0)
            e = ++g_epoch;  // 0 never tags a word (a fresh workspace may hold zeros)
        ka.epoch = e;
        ka.Rg = s.Rg;
        ka.W = s.W;
    }
    ka.PF = s.PF;

    CUtensorMap tmk, tmv;
    const bool swz = s.engine == art::kEngineMma;
    if ((st = make_cache_map(&tmk, &p->k_cache, pr.dtype, swz)) != ART_OK)
        return st;
    if ((st = make_cache_map(&tmv, &p->v_cache, pr.dtype, swz)) != ART_OK)
        return st;

    const int units = pr.B * pr.Hkv;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = s.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(units * s.C);
    cfg.blockDim = dim3(s.threads);
    cfg.dynamicSmemBytes = s.smem;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (gr) {
        // no clusters; every CTA resident at once (they wait on one another)
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    }
    if (p->info) {
        p->info->engine = s.engine;
        p->info->cluster_size = s.C;
        p->info->grid = units * s.C;
        p->info->threads = s.threads;
        p->info->stages = s.S;
        p->info->compute_warps = s.NW;
        p->info->window = s.RF;
        p->info->ring_slots = gr ? s.Rg : s.R;
        p->info->prefetch = s.PF;
        p->info->smem_bytes = s.smem;
        p->info->merge_cta = s.dl;
    }
    if (cudaLaunchKernelEx(&cfg, fn, ka, tmk, tmv) != cudaSuccess) {
        cudaGetLastError();
        return ART_ERR_LAUNCH;
    }
    return ART_OK;
}

}  // namespace

namespace art_host {

int64_t gr_min_workspace_bytes(const art_params_t *p)
{
    if (!p)
        return ART_ERR_NULL;
    Problem pr;
    art_status_t st = check_tensors(p, &pr);
    if (st != ART_OK)
        return st;
    if ((st = check_params(p)) != ART_OK)
        return st;
    DeviceInfo di;
    if ((st = device_info(&di)) != ART_OK)
        return st;
    // any non-null workspace without a size limit: choose_gr then settles the
    // launch shape (it never dereferences the pointer)
    art_params_t q = *p;
    q.merge_cta = 2;
    q.workspace = reinterpret_cast<void *>(static_cast<uintptr_t>(256));
    q.workspace_bytes = INT64_MAX;
    Shape s;
    bool chosen = false;
    int64_t need = 0;
    if ((st = choose_gr(&q, pr, di, &s, &chosen, &need)) != ART_OK)
        return st;
    if (!chosen)
        return 0;
    const uint32_t slot =
        art::make_dl_layout(0, s.R, pr.page, pr.d, (int)elem_size(pr.dtype), s.gmax, s.R).slot_bytes;
    return art::gr_workspace_bytes(pr.B * pr.Hkv, s.W, 16, slot);
}

}  // namespace art_host

extern "C" {

art_status_t art_decode_attention_ex(const art_params_t *p, art_stream_t stream)
{
    if (!p)
        return ART_ERR_NULL;
    return launch(p, stream);
}

int64_t art_workspace_bytes(const art_params_t *p)
{
    if (!p)
        return ART_ERR_NULL;
    Problem pr;
    art_status_t st = check_tensors(p, &pr);
    if (st != ART_OK)
        return st;
    if ((st = check_params(p)) != ART_OK)
        return st;
    DeviceInfo di;
    if ((st = device_info(&di)) != ART_OK)
        return st;
    if (p->merge_cta == -1 || p->merge_cta == 1 || (p->merge_cta != 2 && pr.B * pr.Hkv >= di.sms))
        return 0;
    art_params_t q = *p;
    q.merge_cta = 2;
    q.workspace = nullptr;
    Shape s;
    bool chosen = false;
    int64_t need = 0;
    choose_gr(&q, pr, di, &s, &chosen, &need);
    return need;
}

art_status_t art_decode_attention_multi(const art_params_t *p, int32_t n_queries, art_stream_t stream)
{
    if (!p)
        return ART_ERR_NULL;
    if (n_queries != 1 && n_queries != 2)
        return ART_ERR_UNSUPPORTED;
    return launch(p, stream, n_queries, true);
}

art_status_t art_decode_attention(const art_tensor_t *q, const art_tensor_t *k_cache, const art_tensor_t *v_cache,
                                  const art_tensor_t *page_table, const art_tensor_t *block_order,
                                  const art_tensor_t *seq_lens, float eps_m, float eps_d, int32_t P,
                                  int32_t min_blocks, art_tensor_t *out, art_tensor_t *stop_block,
                                  art_stream_t stream)
{
    if (!q || !k_cache || !v_cache || !page_table || !seq_lens || !out || !stop_block)
        return ART_ERR_NULL;
    art_params_t p;
    std::memset(&p, 0, sizeof p);
    p.q = *q;
    p.k_cache = *k_cache;
    p.v_cache = *v_cache;
    p.page_table = *page_table;
    if (block_order)
        p.block_order = *block_order;  // else zeroed: the default order
    p.seq_lens = *seq_lens;
    p.out = *out;
    p.stop_block = *stop_block;
    p.eps_m = eps_m;
    p.eps_d = eps_d;
    p.P = P;
    p.min_blocks = min_blocks;
    return launch(&p, stream);
}

art_status_t art_build_order_sink_recency(const art_tensor_t *seq_lens, int32_t page, art_tensor_t *block_order,
                                          art_stream_t stream)
{
    if (is_null(seq_lens) || is_null(block_order))
        return ART_ERR_NULL;
    if (seq_lens->ndim != 1 || block_order->ndim != 2 || seq_lens->dtype != ART_I32 ||
        block_order->dtype != ART_I32)
        return seq_lens->ndim != 1 || block_order->ndim != 2 ? ART_ERR_SHAPE : ART_ERR_DTYPE;
    const int64_t B = seq_lens->shape[0];
    if (B <= 0 || B > 65535 || block_order->shape[0] != B || block_order->shape[1] <= 0 ||
        block_order->shape[1] > (int64_t)INT32_MAX || seq_lens->stride[0] != 1 || block_order->stride[1] != 1 ||
        block_order->stride[0] < block_order->shape[1])
        return ART_ERR_SHAPE;
    if (page <= 0)
        return ART_ERR_PARAM;
    if (!aligned(seq_lens->data, 4) || !aligned(block_order->data, 4))
        return ART_ERR_SHAPE;
    const int mb = (int)block_order->shape[1];
    const int threads = 256;
    int gx = (mb + threads - 1) / threads;
    gx = gx > 64 ? 64 : gx;
    art_build_order_kernel<<<dim3(gx, (unsigned)B), threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const int32_t *>(seq_lens->data), (int)B, page, static_cast<int32_t *>(block_order->data),
        block_order->stride[0], mb);
    if (cudaGetLastError() != cudaSuccess)
        return ART_ERR_LAUNCH;
    return ART_OK;
}

const char *art_strerror(art_status_t s)
{
    switch (s) {
    case ART_OK: return "success";
    case ART_ERR_NULL: return "a required pointer is NULL";
    case ART_ERR_SHAPE: return "inconsistent shapes, strides or alignment";
    case ART_ERR_DTYPE: return "wrong or mismatched element type";
    case ART_ERR_UNSUPPORTED: return "head dim, page size or group size not supported";
    case ART_ERR_PARAM: return "invalid threshold, patience, min_blocks or option";
    case ART_ERR_LAUNCH: return "the CUDA runtime refused the launch";
    case ART_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
    case ART_ERR_BAD_INDEX: return "an order or page-table entry, or a sequence length, is out of range";
    case ART_ERR_SCRATCH_SIZE: return "the problem needs more scratch memory than the library's fixed array holds";
    }
    return "unknown status";
}

int32_t art_version(void) { return 100; }

}  // extern "C"
