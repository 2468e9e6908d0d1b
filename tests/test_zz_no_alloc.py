"""The no-allocation routing entry point (tk_gating_route_static), called
through the C ABI, against the allocating one (tk_gating_route) on the same
inputs, two calls in a row each.  Collected last (file name) so that it also
runs after every other GPU test; it passes alone in a fresh process too."""
import numpy as np
import pytest
import torch

import moe_router_gating_b200 as tk
import workloads

pytestmark = pytest.mark.gpu

SENTINEL = -7


def _outputs(T, k, E):
    return [torch.full((m,), SENTINEL, dtype=torch.int32, device="cuda") for m in (E + 1, T * k, T * k)]


def _call(fn, d_ids, T, k, E, stream=0):
    off, ss, sp = _outputs(T, k, E)
    st = fn(d_ids.data_ptr(), T, k, E, off.data_ptr(), ss.data_ptr(), sp.data_ptr(), stream)
    torch.cuda.synchronize()
    return st, off.cpu().numpy(), ss.cpu().numpy(), sp.cpu().numpy()


@pytest.mark.parametrize("T,k,E,kind", [(65536, 8, 256, "skew"), (4096, 8, 256, "uniform"),
                                        (60000, 16, 440, "uniform"), (300, 3, 64, "uniform"), (1, 8, 256, "uniform")])
def test_static_scratch_matches_allocating_entry_point(T, k, E, kind):
    d_ids = torch.from_numpy(workloads.expert_ids(T, k, E, seed=T + E, kind=kind)).cuda()
    st, *ref = _call(tk.route_ptr, d_ids, T, k, E)
    assert st == tk.TK_OK
    for _ in range(2):  # two calls in a row reuse the same scratch
        st, *out = _call(tk.route_static_ptr, d_ids, T, k, E)
        assert st == tk.TK_OK, tk.status_string(st)
        for a, b in zip(out, ref):  # integers: the tolerance is zero
            assert np.array_equal(a, b)


def test_static_scratch_back_to_back_on_one_stream():
    # two calls queued on one stream without a host synchronisation between them
    T, k, E = 65536, 8, 256
    ids_a = torch.from_numpy(workloads.expert_ids(T, k, E, seed=1)).cuda()
    ids_b = torch.from_numpy(workloads.expert_ids(T, k, E, seed=2, kind="skew")).cuda()
    ref = [_call(tk.route_ptr, d, T, k, E)[1:] for d in (ids_a, ids_b)]
    outs = [_outputs(T, k, E) for _ in range(2)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())  # the sentinel fills and the ids land first
    for d, (off, ss, sp) in zip((ids_a, ids_b), outs):
        assert tk.route_static_ptr(d.data_ptr(), T, k, E, off.data_ptr(), ss.data_ptr(), sp.data_ptr(),
                                   s.cuda_stream) == tk.TK_OK
    torch.cuda.synchronize()
    for r, o in zip(ref, outs):
        for a, b in zip(o, r):
            assert np.array_equal(a.cpu().numpy(), b)


def test_static_scratch_rejects_what_does_not_fit():
    # E = 1024 over 128 CTAs needs 512 KiB of counts, more than the 256 KiB array
    T, k, E = 65536, 8, 1024
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert tk.route_plan(T, k, E, sms)["workspace_bytes"] > 256 * 1024
    d_ids = torch.from_numpy(workloads.expert_ids(T, k, E, seed=3)).cuda()
    st, off, ss, sp = _call(tk.route_static_ptr, d_ids, T, k, E)
    assert st == tk.TK_ERR_UNSUPPORTED
    assert (off == SENTINEL).all() and (ss == SENTINEL).all() and (sp == SENTINEL).all()
