"""ra_decode_step_static: the decode step for callers that cannot allocate device memory.

Such callers (a plugin that its engine gives only input/output pointers, a serving loop that
bans cudaMalloc after start-up) call the variant that runs on libra's built-in 64 MiB scratch.
These tests call it through the C ABI and hold it to the workspace entry point's results with
the parity tolerances, on two calls in a row (the second call reuses the scratch the first one
left behind).  This file is collected last on purpose.
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
def test_static_variant_matches_the_workspace_entry_point_twice_in_a_row():
    import torch

    from gpu_util import cache_from_workload, to_dev_bf16
    from parity import check_out
    from synth import gen

    w = gen.workload("l8b_128k_k1pct")          # needs about 48 MiB of scratch
    need = ra.ra_decode_workspace_bytes(w.B, w.Hq, w.N, w.d, w.k, w.n_sink, w.n_window)
    assert 0 < need <= 64 << 20
    cache, q0, _ = cache_from_workload(w)
    q1 = to_dev_bf16(gen.gen_q(w.seed + 1, w.B, w.Hq, w.d))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for q in (q0, q1):                          # two calls in a row on the shared scratch
        out_s = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
        idx_s = torch.full((w.B, w.Hq, w.k), -7, dtype=torch.int32, device="cuda")
        st = ra.ra_decode_step_static(cache.kv, q.data_ptr(), w.Hq, w.k, w.n_sink, w.n_window,
                                      out_s.data_ptr(), idx_s.data_ptr(), stream)
        assert st == ra.RA_OK, ra.ra_status_str(st)
        out_w, idx_w = ra.decode_step(cache, q, w.k, w.n_sink, w.n_window)
        torch.cuda.synchronize()
        check_out(out_s.cpu().numpy(), out_w.cpu().numpy(), "static vs workspace")
        a = np.sort(idx_s.cpu().numpy(), axis=-1)
        b = np.sort(idx_w.cpu().numpy(), axis=-1)
        assert np.array_equal(a, b)
