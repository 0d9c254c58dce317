"""Child process of test_zz_no_alloc.py::test_noalloc_follows_a_device_reset.

Runs with ONE CUDA runtime in the process: the shared libcudart that the
dynamically linked build of the library also uses (torch is not imported, it
would bring a runtime of its own).  So cudaDeviceReset below re-creates the
very context the library's kernels live in, and the library's next call has
to find its scratch array at its new address.

    python noalloc_reset_child.py <libcudart.so> <libexattn (cudart=shared)>

Steps: forward, then the workspace backward (reference) and attn_bwd_noalloc
on the same inputs; cudaDeviceReset; the same inputs again, forward and
attn_bwd_noalloc.  Prints one JSON line with the largest relative-to-max
difference of each gradient from the reference, before and after the reset.
"""
import ctypes
import json
import sys

import numpy as np

B, H, N, D = 1, 4, 1000, 128
CAUSAL = 1
SCALE = 1.0 / np.sqrt(D)


def to_bf16_bits(x):
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def from_bf16_bits(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def main():
    rt = ctypes.CDLL(sys.argv[1], mode=ctypes.RTLD_GLOBAL)
    lib = ctypes.CDLL(sys.argv[2])
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    rt.cudaMalloc.argtypes = [ctypes.POINTER(vp), sz]
    rt.cudaFree.argtypes = [vp]
    rt.cudaMemcpy.argtypes = [vp, vp, sz, i]
    rt.cudaDeviceSynchronize.argtypes = []
    rt.cudaDeviceReset.argtypes = []
    lib.attn_fwd.argtypes = [vp] * 5 + [i] * 4 + [f, i, vp]
    lib.attn_bwd.argtypes = [vp] * 9 + [i] * 4 + [f, i, vp, sz, vp]
    lib.attn_bwd_workspace_bytes.argtypes = [i] * 4
    lib.attn_bwd_workspace_bytes.restype = sz
    lib.attn_bwd_noalloc.argtypes = [vp] * 9 + [i] * 4 + [f, i, vp]
    lib.attn_get_device_status.argtypes = [vp]

    def ok(e, what):
        if e != 0:
            raise SystemExit(f"{what} returned {e}")

    rng = np.random.default_rng(7)
    host = {n: to_bf16_bits(rng.standard_normal((B, H, N, D), dtype=np.float32)) for n in ("q", "k", "v", "do")}
    tbytes = B * H * N * D * 2

    def alloc(nbytes):
        p = vp()
        ok(rt.cudaMalloc(ctypes.byref(p), nbytes), "cudaMalloc")
        return p

    def upload():
        d = {}
        for n, a in host.items():
            d[n] = alloc(tbytes)
            ok(rt.cudaMemcpy(d[n], a.ctypes.data, tbytes, 1), "cudaMemcpy H2D")
        for n in ("o", "dq", "dk", "dv"):
            d[n] = alloc(tbytes)
        d["lse"] = alloc(B * H * N * 4)
        return d

    def download(p):
        a = np.empty((B, H, N, D), dtype=np.uint16)
        ok(rt.cudaMemcpy(a.ctypes.data, p, tbytes, 2), "cudaMemcpy D2H")
        return from_bf16_bits(a).astype(np.float64)

    def forward(d):
        ok(lib.attn_fwd(d["q"], d["k"], d["v"], d["o"], d["lse"], B, H, N, D, SCALE, CAUSAL, None), "attn_fwd")

    def noalloc(d):
        ok(lib.attn_bwd_noalloc(d["q"], d["k"], d["v"], d["o"], d["lse"], d["do"], d["dq"], d["dk"], d["dv"],
                                B, H, N, D, SCALE, CAUSAL, None), "attn_bwd_noalloc")
        ok(lib.attn_get_device_status(None), "device status")
        return {n: download(d[n]) for n in ("dq", "dk", "dv")}

    d = upload()
    forward(d)
    ws_bytes = lib.attn_bwd_workspace_bytes(B, H, N, D)
    ws = alloc(ws_bytes)
    ok(lib.attn_bwd(d["q"], d["k"], d["v"], d["o"], d["lse"], d["do"], d["dq"], d["dk"], d["dv"], B, H, N, D,
                    SCALE, CAUSAL, ws, ws_bytes, None), "attn_bwd")
    ok(lib.attn_get_device_status(None), "device status")
    ref = {n: download(d[n]) for n in ("dq", "dk", "dv")}
    before = noalloc(d)

    ok(rt.cudaDeviceSynchronize(), "cudaDeviceSynchronize")
    ok(rt.cudaDeviceReset(), "cudaDeviceReset")  # frees every allocation above

    d = upload()
    forward(d)
    after = noalloc(d)

    def rel(a, b):
        return float(np.max(np.abs(a - b)) / max(float(np.max(np.abs(b))), 1e-3))

    print(json.dumps({"before": {n: rel(before[n], ref[n]) for n in ref},
                      "after": {n: rel(after[n], ref[n]) for n in ref}}))


if __name__ == "__main__":
    main()
