"""Test helper: fill every SM's shared memory with a bit pattern (NaN, -inf)
right before a kernel under test, so that a read of shared memory the kernel
never wrote shows up as a wrong result instead of passing by luck.

The kernel is compiled at run time with NVRTC (cuda-python) and launched on
torch's current stream: one CTA per SM, each writing its whole dynamic
shared memory, nothing else.
"""
import ctypes

import torch

_SRC = r"""
extern "C" __global__ void poison_smem(unsigned int pattern, unsigned int words)
{
    extern __shared__ unsigned int s[];
    volatile unsigned int *v = s;
    for (unsigned int i = threadIdx.x; i < words; i += blockDim.x)
        v[i] = pattern;
    __syncthreads();
}
"""

_state = {}


def _check(res, what):
    err = res[0] if isinstance(res, tuple) else res
    if int(err) != 0:
        raise RuntimeError(f"{what} failed: {err}")
    return res[1:] if isinstance(res, tuple) and len(res) > 1 else None


def _load():
    if "fn" in _state:
        return _state
    from cuda.bindings import driver, nvrtc
    torch.cuda.init()
    torch.cuda.current_stream()          # the primary context is current from here on
    prog, = _check(nvrtc.nvrtcCreateProgram(_SRC.encode(), b"poison.cu", 0, [], []), "nvrtcCreateProgram")
    major, minor = torch.cuda.get_device_capability()
    opts = [f"--gpu-architecture=sm_{major}{minor}a".encode()]
    err, = nvrtc.nvrtcCompileProgram(prog, len(opts), opts)
    if int(err) != 0:
        size, = _check(nvrtc.nvrtcGetProgramLogSize(prog), "log size")
        log = b" " * size
        nvrtc.nvrtcGetProgramLog(prog, log)
        raise RuntimeError(log.decode(errors="replace"))
    size, = _check(nvrtc.nvrtcGetCUBINSize(prog), "cubin size")
    cubin = b" " * size
    _check(nvrtc.nvrtcGetCUBIN(prog, cubin), "cubin")
    import numpy as np
    image = np.char.array(cubin)
    mod, = _check(driver.cuModuleLoadData(image.ctypes.data), "cuModuleLoadData")
    fn, = _check(driver.cuModuleGetFunction(mod, b"poison_smem"), "cuModuleGetFunction")
    dev = torch.cuda.current_device()
    smem = torch.cuda.get_device_properties(dev).shared_memory_per_block_optin
    _check(driver.cuFuncSetAttribute(
        fn, driver.CUfunction_attribute.CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES, smem), "smem attribute")
    _state.update(driver=driver, mod=mod, fn=fn, smem=smem, image=image,
                  sms=torch.cuda.get_device_properties(dev).multi_processor_count)
    return _state


def poison(pattern: int) -> None:
    """Write the 32-bit pattern over all shared memory of every SM (one
    launch on the current stream, synchronised before returning)."""
    st = _load()
    driver = st["driver"]
    words = st["smem"] // 4
    params = ((pattern & 0xFFFFFFFF, words), (ctypes.c_uint, ctypes.c_uint))
    stream = driver.CUstream(torch.cuda.current_stream().cuda_stream)
    _check(driver.cuLaunchKernel(st["fn"], st["sms"], 1, 1, 1024, 1, 1, st["smem"], stream, params, 0),
           "cuLaunchKernel")
    torch.cuda.synchronize()


NAN = 0x7FC00000
NEG_INF = 0xFF800000
