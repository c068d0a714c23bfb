"""The library-owned workspace (params->workspace == NULL): it grows in
stream order on the call's stream, and a call under stream capture that
would need it to grow is refused with PDA_ERR_WORKSPACE instead."""

import pytest
import torch

from paged_kv_decode_30_b200 import binding as B
from paged_kv_decode_30_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

CASE = W.Workload(name="library_ws", batch=16, num_q_heads=32, num_kv_heads=8, head_dim=128,
                  page_size=16, kv_lens=("uniform", 300, 2500), seed=51)


def _call(t, wl, splits, out, lse, stream):
    return B.paged_decode_attn(t["q"], t["k_pages"], t["v_pages"], t["page_table"],
                               t["kv_lens"], num_kv_heads=wl.num_kv_heads, scale=W.scale_of(wl),
                               num_splits=splits, out=out, lse=lse, stream=stream,
                               library_workspace=True)


def test_library_workspace_grows_on_a_side_stream_and_refuses_growth_under_capture():
    inp = W.generate(CASE)
    t = U.to_device(inp)
    ref_out, ref_lse = U.run_oracle(inp)
    wl = CASE
    out = torch.empty((wl.batch, 1, wl.num_q_heads, wl.head_dim), dtype=torch.float32,
                      device="cuda")
    lse = torch.empty((wl.batch, 1, wl.num_q_heads), dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream()
    # growing calls (each needs more than the last) queued back to back on a
    # non-default stream, with no host synchronisation between them
    results = []
    with torch.cuda.stream(side):
        for splits in (2, 5, 11):
            o = torch.full_like(out, float("nan"))
            l_ = torch.full_like(lse, float("nan"))
            _, _, used = _call(t, wl, splits, o, l_, side)
            assert used == splits
            results.append((o, l_, splits))
    side.synchronize()
    assert B.last_device_error() == 0
    for o, l_, splits in results:
        U.assert_parity(o.double().cpu().numpy(), l_.double().cpu().numpy(), ref_out, ref_lse,
                        W.KV_BF16, f"library workspace, s={splits}")

    # under capture: a call that fits the grown buffer is captured and
    # replays correctly; one that needs more is refused
    g = torch.cuda.CUDAGraph()
    refused = None
    with torch.cuda.graph(g):
        cap = torch.cuda.current_stream()
        _call(t, wl, 11, out, lse, cap)
        try:
            _call(t, wl, 64, out, lse, cap)
        except B.PdaError as e:
            refused = e.status
    assert refused == 4  # PDA_ERR_WORKSPACE
    for _ in range(3):
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert B.last_device_error() == 0
        U.assert_parity(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out,
                        ref_lse, W.KV_BF16, "library workspace, graph replay")
    del g
    # outside capture the same call grows the buffer and runs
    _, _, used = _call(t, wl, 64, out, lse, None)
    torch.cuda.synchronize()
    assert B.last_device_error() == 0
    U.assert_parity(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out, ref_lse,
                    W.KV_BF16, f"library workspace, s={used}")
