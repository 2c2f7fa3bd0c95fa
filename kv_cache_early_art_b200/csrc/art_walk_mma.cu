// art_walk_mma.cu -- walk kernel instantiations for bf16 caches on the
// tensor-core block engine.
#include "art_walk.h"
#include "art_walk_dl.cuh"
#include "art_walk_gr.cuh"

namespace art_walk {

namespace {
template <int GMAX, int NMW>
KernelFn by_dp(int d, int page)
{
    using art::art_walk_kernel;
    using T = __nv_bfloat16;
    constexpr int E = art::kEngineMma;
    if (d == 64)
        return page == 16 ? art_walk_kernel<T, 64, 16, GMAX, E, NMW> : art_walk_kernel<T, 64, 64, GMAX, E, NMW>;
    return page == 16 ? art_walk_kernel<T, 128, 16, GMAX, E, NMW> : art_walk_kernel<T, 128, 64, GMAX, E, NMW>;
}
}  // namespace

KernelFn bf16_mma(int gmax, int nmw, int d, int page, bool detector)
{
    using art::art_walk_kernel;
    using T = __nv_bfloat16;
    constexpr int E = art::kEngineMma;
    if (!detector) {
        // the detector-off reference exists for d = 128, 64-token pages
        if (d != 128 || page != 64)
            return nullptr;
        if (nmw == 4)
            return gmax == 4 ? art_walk_kernel<T, 128, 64, 4, E, 4, 1, false>
                             : art_walk_kernel<T, 128, 64, 8, E, 4, 1, false>;
        return gmax == 4 ? art_walk_kernel<T, 128, 64, 4, E, 1, 1, false> : art_walk_kernel<T, 128, 64, 8, E, 1, 1, false>;
    }
    if (nmw == 4)
        return gmax == 4 ? by_dp<4, 4>(d, page) : by_dp<8, 4>(d, page);
    return gmax == 4 ? by_dp<4, 1>(d, page) : by_dp<8, 1>(d, page);
}

KernelFn bf16_mma_dl(int gmax, int d, int page, bool detector)
{
    using art::art_walk_dl_kernel;
    using T = __nv_bfloat16;
    constexpr int E = art::kEngineMma;
    if (d != 128 || page != 64)
        return nullptr;
    if (detector)
        return gmax == 4 ? art_walk_dl_kernel<T, 128, 64, 4, E, 4, true> : art_walk_dl_kernel<T, 128, 64, 8, E, 8, true>;
    return gmax == 4 ? art_walk_dl_kernel<T, 128, 64, 4, E, 4, false> : art_walk_dl_kernel<T, 128, 64, 8, E, 8, false>;
}

KernelFn bf16_mma_gr(int gmax, int d, int page, bool detector)
{
    using art::art_walk_gr_kernel;
    using T = __nv_bfloat16;
    constexpr int E = art::kEngineMma;
    if (d != 128 || page != 64)
        return nullptr;
    if (detector)
        return gmax == 4 ? art_walk_gr_kernel<T, 128, 64, 4, E, 4, true> : art_walk_gr_kernel<T, 128, 64, 8, E, 8, true>;
    return gmax == 4 ? art_walk_gr_kernel<T, 128, 64, 4, E, 4, false> : art_walk_gr_kernel<T, 128, 64, 8, E, 8, false>;
}

}  // namespace art_walk
