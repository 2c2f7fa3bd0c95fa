// art_walk_multi.cu -- walk kernel instantiations for two query tokens of a
// sequence sharing one walk (head dim 128).
#include "art_walk.h"

namespace art_walk {

namespace {
template <typename T, int ENGINE, int GMAX, int NMW>
KernelFn by_page(int page)
{
    return page == 16 ? art::art_walk_kernel<T, 128, 16, GMAX, ENGINE, NMW, 2>
                      : art::art_walk_kernel<T, 128, 64, GMAX, ENGINE, NMW, 2>;
}
}  // namespace

KernelFn multi(bool f32, int engine, int page, int gmax, int nmw)
{
    if (f32)
        return gmax == 4 ? by_page<float, art::kEngineCuda, 4, 1>(page) : by_page<float, art::kEngineCuda, 8, 1>(page);
    if (engine != art::kEngineMma)
        return nullptr;
    using T = __nv_bfloat16;
    if (nmw == 4)
        return gmax == 4 ? by_page<T, art::kEngineMma, 4, 4>(page) : by_page<T, art::kEngineMma, 8, 4>(page);
    return gmax == 4 ? by_page<T, art::kEngineMma, 4, 1>(page) : by_page<T, art::kEngineMma, 8, 1>(page);
}

}  // namespace art_walk
