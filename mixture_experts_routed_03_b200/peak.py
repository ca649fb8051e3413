"""ctypes binding of the tensor-core peak probe (``libmoe_peak.so``): the
dense tcgen05 MMA rate of this GPU per operand kind and tile shape, against
which the benchmark states its roofline fractions.  A measurement tool, not
part of the layer."""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_peak.so")
KINDS = {"bf16": 0, "fp8": 1, "nvfp4": 2, "mxfp8": 3}
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run python -m mixture_experts_routed_03_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        L.moe_peak_mma.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]
        L.moe_peak_mma.restype = ctypes.c_int
        _lib = L
    return _lib


def mma_peak(kind, n=256, pair=False, iters=20000, stream=None):
    """(TFLOP/s over all SMs, SM cycles per MMA instruction) of back-to-back
    tcgen05.mma of `kind` ('bf16', 'fp8', 'nvfp4') with N = n, M = 128 per CTA
    or 256 per CTA pair (pair=True, cta_group::2)."""
    import torch
    scratch = torch.zeros(4096, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    tf, cyc = ctypes.c_float(0.0), ctypes.c_float(0.0)
    rc = lib().moe_peak_mma(KINDS[kind], int(n), int(bool(pair)), int(iters), scratch.data_ptr(), st,
                            ctypes.byref(tf), ctypes.byref(cyc))
    if rc != 0:
        raise RuntimeError(f"moe_peak_mma({kind}, n={n}, pair={pair}) returned {rc}")
    return float(tf.value), float(cyc.value)


def mainloop(pair=False, mma=True, iters=4000, src_bytes=32 << 20, stream=None):
    """(SM cycles per K block, aggregate GB/s into shared memory) of the
    grouped GEMMs' operand feed: 4-stage bulk-copy ring of 128-row A and
    256-row B K blocks (one CTA, or halves in a CTA pair) from a src_bytes
    source, with (mma=True) or without the E4M3 MMAs of each block."""
    import torch
    L = lib()
    L.moe_peak_mainloop.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_longlong,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_float),
                                    ctypes.POINTER(ctypes.c_float)]
    L.moe_peak_mainloop.restype = ctypes.c_int
    src = torch.zeros(src_bytes, dtype=torch.uint8, device="cuda")
    scratch = torch.zeros(4096, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    cyc, gbs = ctypes.c_float(0.0), ctypes.c_float(0.0)
    rc = L.moe_peak_mainloop(int(bool(pair)), int(bool(mma)), int(iters), src.data_ptr(), src_bytes,
                             scratch.data_ptr(), st, ctypes.byref(cyc), ctypes.byref(gbs))
    if rc != 0:
        raise RuntimeError(f"moe_peak_mainloop(pair={pair}, mma={mma}) returned {rc}")
    return float(cyc.value), float(gbs.value)


def tmem_read(warps=8, loads=1, iters=2000):
    """Bytes per SM cycle from tensor memory to registers (one CTA, `warps`
    warps, `loads` 16-column tcgen05.ld in flight per wait)."""
    import torch
    L = lib()
    L.moe_peak_tmem_read.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.POINTER(ctypes.c_float)]
    L.moe_peak_tmem_read.restype = ctypes.c_int
    scratch = torch.zeros(64, dtype=torch.int32, device="cuda")
    bpc = ctypes.c_float(0.0)
    rc = L.moe_peak_tmem_read(int(warps), int(loads), int(iters), scratch.data_ptr(),
                              torch.cuda.current_stream().cuda_stream, ctypes.byref(bpc))
    if rc != 0:
        raise RuntimeError(f"moe_peak_tmem_read returned {rc}")
    return float(bpc.value)
