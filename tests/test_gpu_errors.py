"""Device-side error reporting, exercised without faulting the GPU: every
bad input here is one that the kernels check before the access it guards,
and every wait is bounded.  The error word carries the first code set; the
context stays usable afterwards (a normal call follows each case)."""
import numpy as np
import pytest
import torch

import oracle as O
from workload import CONFIGS, make_hidden_states, make_weights

pytestmark = pytest.mark.gpu

F = pytest.importorskip("cross_loop_sparse_b200.flashloop")
from gpu_helpers import bf16_to_torch, i32  # noqa: E402

DEVERR_CAPACITY, DEVERR_INDEX, DEVERR_TIMEOUT, DEVERR_RANGE = 1, 2, 3, 4


def _gate_case():
    cfg = CONFIGS["tiny"]
    X, _ = make_hidden_states(cfg)
    p = F.Params.from_config(cfg)
    st = F.FlashLoopState(p, kv_only=True)
    return cfg, X, p, st


def _run_gate(p, st, xc, xp, prev, nprev, prev_cap, out_cap, S):
    act = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    slot = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    st["err"].zero_()
    F.flashloop_gate(p, xc, xp, prev, nprev, prev_cap, act, slot, n, out_cap, st["workspace"], st["err"])
    code = st.error_code()
    return code, int(n.item()), act.cpu().numpy(), slot.cpu().numpy()


def test_gate_capacity_overflow_truncates_and_reports():
    """More active tokens than the output capacity: the first out_capacity
    of the ascending list are written, the count is the capacity, and the
    error word says FLASHLOOP_DEVERR_CAPACITY."""
    cfg, X, p, st = _gate_case()
    S = cfg.seq
    xs = [bf16_to_torch(x) for x in X]
    want = O.gate(X[1], X[0], np.arange(S), cfg.tau)
    cap = want.size // 2
    code, n, act, slot = _run_gate(p, st, xs[1], xs[0], None, None, S, cap, S)
    assert code == DEVERR_CAPACITY
    assert n == cap
    assert np.array_equal(act[:cap], want[:cap])
    ws = np.full(S, -1, np.int32)
    ws[want[:cap]] = np.arange(cap)
    assert np.array_equal(slot, ws)
    code, n, act, _ = _run_gate(p, st, xs[1], xs[0], None, None, S, S, S)   # still usable
    assert code == 0 and n == want.size and np.array_equal(act[:n], want)


def test_gate_candidate_index_out_of_range_is_reported_not_loaded():
    """A candidate token >= S (or < 0) is refused before its row is read: the
    error word says FLASHLOOP_DEVERR_INDEX and the other candidates are gated
    as usual."""
    cfg, X, p, st = _gate_case()
    S = cfg.seq
    xs = [bf16_to_torch(x) for x in X]
    prev = O.gate(X[1], X[0], np.arange(S), cfg.tau)
    bad = prev.copy()
    bad[3] = S + 1000
    bad[7] = -5
    code, n, act, _ = _run_gate(p, st, xs[2], xs[1], i32(bad), i32([bad.size]), S, S, S)
    assert code == DEVERR_INDEX
    keep = np.delete(prev, [3, 7])
    want = O.gate(X[2], X[1], keep, cfg.tau)
    assert n == want.size and np.array_equal(act[:n], want)


@pytest.mark.parametrize("kind", [0, 1])
def test_bounded_wait_gives_up_and_reports(kind):
    """The spinning (0) and sleeping (1) barrier waits of the pipelined
    kernels, on a barrier that never completes: the kernel returns with
    FLASHLOOP_DEVERR_TIMEOUT in the error word instead of hanging."""
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    F.flashloop_selftest_bounded_wait(kind, err)
    torch.cuda.synchronize()
    assert int(err.item()) == DEVERR_TIMEOUT
    cfg, X, p, st = _gate_case()       # the context is still usable
    xs = [bf16_to_torch(x) for x in X]
    code, n, _, _ = _run_gate(p, st, xs[1], xs[0], None, None, cfg.seq, cfg.seq, cfg.seq)
    assert code == 0 and n == O.gate(X[1], X[0], np.arange(cfg.seq), cfg.tau).size


def test_fp16_range_of_attention_operands_is_checked():
    """Hidden states scaled so that the keys and queries exceed fp16's range
    (the tensor-core operand type): the loop-1 step reports
    FLASHLOOP_DEVERR_RANGE; the same step on the unscaled input reports
    nothing."""
    cfg = CONFIGS["tiny"]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    p = F.Params.from_config(cfg)
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    for scale, want in ((1.0, 0), (2.0 ** 20, DEVERR_RANGE)):
        st = F.FlashLoopState(p)
        x = bf16_to_torch(X[0]).float() * scale
        F.flashloop_loop_step(p, 1, x.to(torch.bfloat16).contiguous(), None, wqkv, wo, st)
        assert st.error_code() == want, scale
