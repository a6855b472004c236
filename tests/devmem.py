"""Device-memory readings for the tests, through the CUDA driver API (ctypes):
free device memory, and the used-memory high-water mark of the device's
default memory pool -- the pool that stream-ordered allocation
(cudaMallocAsync) draws from.  Resetting the mark to 0 before a call and
reading it after shows whether the call took any memory from that pool."""
import ctypes

_CU_MEMPOOL_ATTR_USED_MEM_HIGH = 8


def _driver():
    lib = ctypes.CDLL("libcuda.so.1")
    lib.cuDeviceGet.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_int]
    lib.cuDeviceGetDefaultMemPool.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
    lib.cuMemPoolGetAttribute.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    lib.cuMemPoolSetAttribute.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    lib.cuMemGetInfo_v2.argtypes = [ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]
    return lib


def _pool(ordinal: int):
    lib = _driver()
    dev = ctypes.c_int()
    assert lib.cuDeviceGet(ctypes.byref(dev), ordinal) == 0
    pool = ctypes.c_void_p()
    assert lib.cuDeviceGetDefaultMemPool(ctypes.byref(pool), dev.value) == 0
    return lib, pool


def reset_pool_high_water(ordinal: int = 0) -> None:
    lib, pool = _pool(ordinal)
    zero = ctypes.c_uint64(0)
    assert lib.cuMemPoolSetAttribute(pool, _CU_MEMPOOL_ATTR_USED_MEM_HIGH, ctypes.byref(zero)) == 0


def pool_high_water(ordinal: int = 0) -> int:
    lib, pool = _pool(ordinal)
    v = ctypes.c_uint64(0)
    assert lib.cuMemPoolGetAttribute(pool, _CU_MEMPOOL_ATTR_USED_MEM_HIGH, ctypes.byref(v)) == 0
    return v.value


def free_bytes() -> int:
    """Free memory of the current context's device."""
    lib = _driver()
    free, total = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.cuMemGetInfo_v2(ctypes.byref(free), ctypes.byref(total)) == 0
    return free.value
