"""Checkpoint and resume of the loop state.

The whole state of a sequence lives in caller-owned device tensors (the KV
streams, active lists and slot maps, the q / m / Z / N slots, column masses,
selections, O, Y, the workspace and the error word).  A checkpoint is those
tensors saved with torch.save; resuming copies them back into the same
buffers (the library holds their addresses).  Saved after loop 2 and loaded
back once loops 3..R have run, loops 3..R run again give the same bytes.

This file is collected after every other test file, so that a
stop-at-first-failure run has already run every other test."""
import numpy as np
import pytest
import torch

from workload import CONFIGS, make_hidden_states, make_weights

pytestmark = pytest.mark.gpu

F = pytest.importorskip("cross_loop_sparse_b200.flashloop")
from gpu_helpers import bf16_to_torch, torch_to_bf16_bits  # noqa: E402


def test_checkpoint_after_loop_2_resumes_byte_for_byte(tmp_path):
    cfg = CONFIGS["tiny"]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    p = F.Params.from_config(cfg)
    st = F.FlashLoopState(p)
    xs = [bf16_to_torch(x) for x in X]
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    F.flashloop_loop_step(p, 1, xs[0], None, wqkv, wo, st)
    F.flashloop_loop_step(p, 2, xs[1], xs[0], wqkv, wo, st)
    torch.cuda.synchronize()
    path = tmp_path / "state_after_loop2.pt"
    torch.save({k: v.cpu() for k, v in st.t.items()}, path)

    def loops_3_to_R():
        for r in range(3, cfg.n_loops + 1):
            F.flashloop_loop_step(p, r, xs[r - 1], xs[r - 2], wqkv, wo, st)
        torch.cuda.synchronize()
        return {k: v.cpu().clone() for k, v in st.t.items()}

    first = loops_3_to_R()
    saved = torch.load(path)
    assert set(saved) == set(st.t)
    for k, v in saved.items():
        st.t[k].copy_(v)
    torch.cuda.synchronize()
    again = loops_3_to_R()
    for name in ("O", "Y"):
        assert np.array_equal(torch_to_bf16_bits(first[name]), torch_to_bf16_bits(again[name])), name
    # every state tensor but the scratch workspace comes back byte for byte
    for k in first:
        if k != "workspace":
            a_bytes = first[k].contiguous().reshape(-1).view(torch.uint8)
            b_bytes = again[k].contiguous().reshape(-1).view(torch.uint8)
            assert torch.equal(a_bytes, b_bytes), k
    assert st.error_code() == 0
