"""ra_decode_step_static: the decode step for callers that cannot allocate device memory.

Such callers (a plugin that its engine gives only input/output pointers, a serving loop that
bans cudaMalloc after start-up) call the variant that runs on libra's built-in 64 MiB scratch.
These tests call it through the C ABI and hold it to the workspace entry point's results with
the parity tolerances, on two calls in a row (the second call reuses the scratch the first one
left behind), then after a call of another shape, and one head of its output to the fp64
oracle.  A first call inside a stream capture is refused (checked in a fresh process, where no
call has looked the scratch up yet).  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import top_retrieval_attention_b200 as ra

FAKE = 1 << 20


def test_static_variant_rejects_shapes_beyond_its_scratch():
    # 32 query heads at N = 2^20 need about 256 MB of workspace: rejected before any launch
    kv = ra.ra_kv(FAKE, FAKE, 1, 8, 128, 1 << 20, 1 << 20)
    need = ra.ra_decode_workspace_bytes(1, 32, 1 << 20, 128, 100, 128, 512)
    assert need > 64 << 20
    s = ra.ra_decode_step_static(kv, FAKE, 32, 100, 128, 512, FAKE, FAKE, None)
    assert s == ra.RA_ERR_WORKSPACE
    # a bad shape is reported like the workspace entry point reports it
    s = ra.ra_decode_step_static(kv, FAKE, 3, 100, 128, 512, FAKE, FAKE, None)
    assert s == ra.RA_ERR_SHAPE


@pytest.mark.gpu
def test_static_variant_matches_the_workspace_entry_point_and_the_oracle():
    import torch

    from gpu_util import cache_from_host, cache_from_workload, to_dev_bf16
    from parity import check_head, check_out
    from synth import gen

    w = gen.workload("l8b_128k_k1pct")          # needs about 48 MiB of scratch
    need = ra.ra_decode_workspace_bytes(w.B, w.Hq, w.N, w.d, w.k, w.n_sink, w.n_window)
    assert 0 < need <= 64 << 20
    cache, q0, nd = cache_from_workload(w)
    q1 = to_dev_bf16(gen.gen_q(w.seed + 1, w.B, w.Hq, w.d))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def static_vs_workspace(c, q, Hq, k, n_sink, n_window):
        B, d = c.B, c.d
        out_s = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
        idx_s = torch.full((B, Hq, k), -7, dtype=torch.int32, device="cuda")
        st = ra.ra_decode_step_static(c.kv, q.data_ptr(), Hq, k, n_sink, n_window,
                                      out_s.data_ptr(), idx_s.data_ptr(), stream)
        assert st == ra.RA_OK, ra.ra_status_str(st)
        out_w, idx_w = ra.decode_step(c, q, k, n_sink, n_window)
        torch.cuda.synchronize()
        out_s, idx_s = out_s.cpu().numpy(), idx_s.cpu().numpy()
        check_out(out_s, out_w.cpu().numpy(), "static vs workspace")
        assert np.array_equal(np.sort(idx_s, axis=-1), np.sort(idx_w.cpu().numpy(), axis=-1))
        return out_s, idx_s

    for q in (q0, q1):                          # two calls in a row on the shared scratch
        static_vs_workspace(cache, q, w.Hq, w.k, w.n_sink, w.n_window)
    # a call of another shape (G = 4, fewer query heads and keys) in between leaves the scratch
    # holding other rows and counts; the next 128K call must not depend on them
    qs, Ks, Vs = (gen.gen_q(77, 1, 8, 128), *gen.host_head(gen.Workload("s", 1, 8, 2, 128, 5000,
                                                                         300, 8, 64, seed=77),
                                                           0, 0, 0, 5000))
    small = cache_from_host(np.stack([Ks, Ks])[None], np.stack([Vs, Vs])[None])
    static_vs_workspace(small, to_dev_bf16(qs), 8, 300, 8, 64)
    out_s, idx_s = static_vs_workspace(cache, q0, w.Hq, w.k, w.n_sink, w.n_window)
    # and the static entry's own output of one head against the fp64 oracle
    qh = gen.gen_q(w.seed, w.B, w.Hq, w.d)
    Kh, Vh = gen.host_head(w, 0, 0, 3, w.N, nd)
    check_head(qh[0, 13], Kh, Vh, w.k, w.n_sink, w.n_window, out_s[0, 13], idx_s[0, 13])


_CAPTURE_CHILD = r"""
import ctypes, sys, torch
sys.path.insert(0, sys.argv[1])
import top_retrieval_attention_b200 as ra
from gpu_util import cache_from_host
import numpy as np
K = np.zeros((1, 1, 700, 128), np.uint16)
c = cache_from_host(K, K)
q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
out = torch.empty((1, 4, 128), dtype=torch.float32, device="cuda")
idx = torch.empty((1, 4, 8), dtype=torch.int32, device="cuda")
s = torch.cuda.Stream()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g, stream=s):
    out.zero_()                     # the capture holds one node either way
    st = ra.ra_decode_step_static(c.kv, q.data_ptr(), 4, 8, 4, 16, out.data_ptr(), idx.data_ptr(),
                                  ctypes.c_void_p(s.cuda_stream))
print("status", st, ra.ra_last_error())
torch.cuda.synchronize()
st2 = ra.ra_decode_step_static(c.kv, q.data_ptr(), 4, 8, 4, 16, out.data_ptr(), idx.data_ptr(),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
torch.cuda.synchronize()
print("after", st2)
"""


@pytest.mark.gpu
def test_static_variant_refuses_a_first_call_inside_a_capture():
    import os
    import subprocess
    import sys
    tests = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(tests)
    env = dict(os.environ, PYTHONPATH=os.pathsep.join([root, tests]))
    r = subprocess.run([sys.executable, "-c", _CAPTURE_CHILD, root], capture_output=True, text=True,
                       env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = r.stdout.splitlines()
    assert any(l.startswith(f"status {ra.RA_ERR_ARG} ") and "before any stream capture" in l
               for l in lines), r.stdout
    assert f"after {ra.RA_OK}" in lines, r.stdout
