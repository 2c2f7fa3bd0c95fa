// art_walk_f32.cu -- walk kernel instantiations for fp32 caches (CUDA-core
// block engine).
#include "art_walk.h"

namespace art_walk {

namespace {
template <int GMAX, bool DET>
KernelFn by_dp(int d, int page)
{
    using art::art_walk_kernel;
    constexpr int E = art::kEngineCuda;
    if (d == 64)
        return page == 16 ? art_walk_kernel<float, 64, 16, GMAX, E, 1, 1, DET>
                          : art_walk_kernel<float, 64, 64, GMAX, E, 1, 1, DET>;
    return page == 16 ? art_walk_kernel<float, 128, 16, GMAX, E, 1, 1, DET>
                      : art_walk_kernel<float, 128, 64, GMAX, E, 1, 1, DET>;
}
}  // namespace

KernelFn f32_cuda(int gmax, int d, int page, bool detector)
{
    if (!detector) {
        // the detector-off reference exists for the small fp32 workload's shape
        if (d != 64 || page != 16 || gmax > 4)
            return nullptr;
        return gmax == 1 ? art::art_walk_kernel<float, 64, 16, 1, art::kEngineCuda, 1, 1, false>
                         : art::art_walk_kernel<float, 64, 16, 4, art::kEngineCuda, 1, 1, false>;
    }
    if (gmax == 1)
        return by_dp<1, true>(d, page);
    return gmax == 4 ? by_dp<4, true>(d, page) : by_dp<8, true>(d, page);
}

}  // namespace art_walk
