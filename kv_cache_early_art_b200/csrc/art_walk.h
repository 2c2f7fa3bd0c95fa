// art_walk.h -- the walk kernel's instantiations, one translation unit per
// group (built in parallel), looked up by the host side of the library.
//
// Each lookup returns the kernel for the given compile-time shape, or NULL
// when that shape is not instantiated.  `detector` false selects the
// instantiation whose merge forms no statistic and never stops (a timing
// reference for the cost of the ART detector; its output equals the eps = 0
// walk's bit for bit).
#pragma once
#include <cuda.h>

#include "art_kernels.cuh"

namespace art_walk {

using KernelFn = void (*)(art::KernelArgs, CUtensorMap, CUtensorMap);

// fp32 caches, CUDA-core block engine (gmax 1, 4 or 8 query rows per unit)
KernelFn f32_cuda(int gmax, int d, int page, bool detector);
// bf16 caches, CUDA-core block engine
KernelFn bf16_cuda(int gmax, int d, int page);
// bf16 caches, tensor-core block engine (gmax 4 or 8; nmw 1 or 4 merge warps)
KernelFn bf16_mma(int gmax, int nmw, int d, int page, bool detector);
// bf16 caches, tensor-core block engine, dedicated merge CTA (gmax 4 or 8)
KernelFn bf16_mma_dl(int gmax, int d, int page, bool detector);
// the same merge reached through a workspace (no clusters, cooperative launch)
KernelFn bf16_mma_gr(int gmax, int d, int page, bool detector);
// two query tokens sharing one walk (head dim 128)
KernelFn multi(bool f32, int engine, int page, int gmax, int nmw);

}  // namespace art_walk
