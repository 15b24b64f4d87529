"""Failure detection without a GPU fault: a pipeline wait that runs out.

nvkv_debug_inject_fault makes the next attention launch's staging producer
skip the first stage, so the converters' wait on it expires (after its 2 s
bound).  The kernel must record NVKV_ERR_TIMEOUT in
the cache's status word, unwind and return (the stream synchronises without
an error), and the next launch, after the caller clears the status and the
workspace, must again be correct.  Nothing traps, faults or hangs."""
import numpy as np
import pytest
import torch

import kvsynth
from oracle.stream import OracleStream
from tests._harness import LibStream, assert_parity, to_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "stream5b"])
def test_expired_wait_reports_status_and_the_context_survives(name):
    import nvfp4_kv_cache_append_b200 as nv
    from nvfp4_kv_cache_append_b200 import _lib as L
    wl = kvsynth.WORKLOADS[name]
    lib = LibStream(wl, nv.NVKV_KV_NVFP4)
    ora = OracleStream(wl, seed=0, keep_inputs=False)
    for step in range(1, 3):
        x = kvsynth.chunk_qkv(wl, step, 0)
        ora.step(k=x["k"], v=x["v"], q=x["q"])
        g = to_gpu(x)
        lib.step(g["q"], g["k"], g["v"])
    torch.cuda.synchronize()
    assert lib.cache.device_status() == 0
    L.nvkv_debug_inject_fault(L.NVKV_FAULT_SKIP_FIRST_STAGE)    # the waits on it end after 2 s
    lib.cache.attention(g["q"])
    torch.cuda.synchronize()                                            # no CUDA error
    assert lib.cache.device_status() == L.STATUS_CODE["NVKV_ERR_TIMEOUT"]
    # the hook was one-shot; the caller clears the status and the workspace
    lib.cache.status.zero_()
    lib.cache.workspace.zero_()
    out = lib.cache.attention(g["q"])
    torch.cuda.synchronize()
    assert lib.cache.device_status() == 0
    got = out.float().cpu().numpy()
    rows = np.unique(np.r_[0, wl.Lq // 3, wl.Lq - 1, np.arange(0, wl.Lq, max(1, wl.Lq // 12))])
    for h in range(0, wl.H, max(1, wl.H // 3)):
        ref, _ = ora.attention(0, h, rows)
        assert_parity(got[0, rows, h], ref, f"after recovery h {h}")
