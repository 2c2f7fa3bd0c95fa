// art_walk_bf16.cu -- walk kernel instantiations for bf16 caches on the
// CUDA-core block engine.
#include "art_walk.h"

namespace art_walk {

namespace {
template <int GMAX>
KernelFn by_dp(int d, int page)
{
    using art::art_walk_kernel;
    using T = __nv_bfloat16;
    constexpr int E = art::kEngineCuda;
    if (d == 64)
        return page == 16 ? art_walk_kernel<T, 64, 16, GMAX, E, 1> : art_walk_kernel<T, 64, 64, GMAX, E, 1>;
    return page == 16 ? art_walk_kernel<T, 128, 16, GMAX, E, 1> : art_walk_kernel<T, 128, 64, GMAX, E, 1>;
}
}  // namespace

KernelFn bf16_cuda(int gmax, int d, int page)
{
    if (gmax == 1)
        return by_dp<1>(d, page);
    return gmax == 4 ? by_dp<4>(d, page) : by_dp<8>(d, page);
}

}  // namespace art_walk
