"""The C ABI library on the CPU: it loads, exports every function the header
declares, its structs have the layout ctypes assumes, and its host-side
checks and sizing helpers answer without a GPU."""
import ctypes
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle as O
from workload import CONFIGS

try:
    from cross_loop_sparse_b200 import flashloop as F
except ImportError as exc:  # pragma: no cover - the library must be built first
    pytest.skip(f"libflashloop.so not built: {exc}", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_every_declared_function_is_exported():
    names = F.header_functions()
    assert len(names) >= 13
    missing = [n for n in names if not hasattr(F._lib, n)]
    assert missing == []


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_struct_layout_matches_header():
    src = r'''
#include <stdio.h>
#include <stddef.h>
#include "flashloop.h"
int main(void) {
  printf("%zu %zu %zu\n", sizeof(flashloop_params), sizeof(flashloop_kv), sizeof(flashloop_state));
  printf("%zu %zu %zu %zu %zu\n", offsetof(flashloop_params, tau), offsetof(flashloop_params, topk),
         offsetof(flashloop_params, capacity), offsetof(flashloop_state, n_active),
         offsetof(flashloop_state, workspace_bytes));
  printf("%zu %zu %zu\n", offsetof(flashloop_state, cols), offsetof(flashloop_state, rope_cs),
         offsetof(flashloop_state, colmass));
  printf("%zu %zu %zu %zu\n", offsetof(flashloop_params, gate_topk), offsetof(flashloop_params, fixed_mass),
         offsetof(flashloop_params, attn_pairs), offsetof(flashloop_state, G));
  printf("%zu %zu %zu %zu %zu\n", offsetof(flashloop_params, kv_scheme), sizeof(flashloop_paper_kv),
         offsetof(flashloop_paper_kv, tail), offsetof(flashloop_state, paper_k), offsetof(flashloop_state, paper_v));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "probe.c")
        exe = os.path.join(d, "probe")
        open(c, "w").write(src)
        subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), c, "-o", exe])
        out = subprocess.check_output([exe], text=True).split()
    got = [int(v) for v in out]
    want = [ctypes.sizeof(F.Params), ctypes.sizeof(F.KV), ctypes.sizeof(F.StateC),
            F.Params.tau.offset, F.Params.topk.offset, F.Params.capacity.offset,
            F.StateC.n_active.offset, F.StateC.workspace_bytes.offset,
            F.StateC.cols.offset, F.StateC.rope_cs.offset, F.StateC.colmass.offset,
            F.Params.gate_topk.offset, F.Params.fixed_mass.offset, F.Params.attn_pairs.offset,
            F.StateC.G.offset, F.Params.kv_scheme.offset, ctypes.sizeof(F.PaperKV), F.PaperKV.tail.offset,
            F.StateC.paper_k.offset, F.StateC.paper_v.offset]
    assert got == want


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k", "prefill_32k", "depth_8k_r8"])
def test_cache_bytes_agree_with_oracle_accounting(name):
    cfg = CONFIGS[name]
    p = F.Params.from_config(cfg)
    n = [cfg.n_active(r) for r in range(1, cfg.n_loops + 1)]
    base, loops = O.cache_bytes(cfg.seq, cfg.n_heads, cfg.head_dim, cfg.bits, n)
    assert F.flashloop_cache_bytes(p, n) == base + sum(loops)


def test_selection_loop_follows_budgets():
    cfg = CONFIGS["tiny"]
    p = F.Params.from_config(cfg)
    assert [F.flashloop_selection_loop(p, r) for r in range(2, 5)] == [2, 2, 2]
    p = F.Params.from_config(cfg, topk=[256, 40, 40, 13])
    assert [F.flashloop_selection_loop(p, r) for r in range(2, 5)] == [2, 2, 4]
    assert F.flashloop_selection_loop(p, 1) == -1


def test_workspace_covers_dense_and_selected_buffers():
    cfg = CONFIGS["prefill_32k"]
    p = F.Params.from_config(cfg)
    S, H, dh = cfg.seq, cfg.n_heads, cfg.head_dim
    assert F.flashloop_workspace_bytes(p) >= 2 * S * H * dh * 4 + 2 * S * H * dh * 2


def _status(p):
    # a parameter error is reported before any device query
    return F._lib.flashloop_rope_table(ctypes.byref(p), 1, None, None)


def test_host_checks_reject_bad_params():
    cfg = CONFIGS["tiny"]
    p = F.Params.from_config(cfg); p.head_dim = 96; p.d_model = 96 * 4
    assert _status(p) == -2
    p = F.Params.from_config(cfg); p.d_model = 200
    assert _status(p) == -1
    p = F.Params.from_config(cfg); p.bits[0] = 4
    assert _status(p) == -2
    p = F.Params.from_config(cfg); p.bits[2] = 3
    assert _status(p) == -2
    p = F.Params.from_config(cfg); p.topk[1] = cfg.seq + 1
    assert _status(p) == -1
    p = F.Params.from_config(cfg, topk=[256, 20, 26, 26])
    assert _status(p) == -1                      # budgets must not grow
    p = F.Params.from_config(cfg); p.capacity[2] = 0
    assert _status(p) == -1
    p = F.Params.from_config(cfg); p.n_loops = 17
    assert _status(p) == -1
    p = F.Params.from_config(cfg); p.attn_pairs = 1  # reserved field
    assert _status(p) == -2
    assert F.flashloop_status_string(-2).startswith("unsupported")


def test_decode_refuses_the_fixed_mass_form():
    """Decode keeps the running (m, N, Z) form: its sizing helper reports the
    fixed-mass parameters as unsupported (0 bytes) before any device query."""
    cfg = CONFIGS["decode_32k"]
    p = F.Params.from_config(cfg)
    assert F._lib.flashloop_decode_workspace_bytes(ctypes.byref(p)) > 0
    p = F.Params.from_config(cfg, fixed_mass=True)
    assert F._lib.flashloop_decode_workspace_bytes(ctypes.byref(p)) == 0


def test_noalloc_gate_refuses_what_the_workspace_gate_refuses():
    """flashloop_gate_noalloc runs flashloop_gate's parameter checks first, so
    bad parameters get the same status from both, before any device query."""
    cfg = CONFIGS["tiny"]
    dummy = ctypes.c_void_p(16)

    def both(p):
        g = F._lib.flashloop_gate(ctypes.byref(p), dummy, dummy, None, None, cfg.seq, dummy, dummy,
                                  dummy, cfg.seq, dummy, dummy, None)
        n = F._lib.flashloop_gate_noalloc(ctypes.byref(p), dummy, dummy, None, None, cfg.seq, dummy,
                                          dummy, dummy, cfg.seq, dummy, None)
        return g, n

    cases = []
    p = F.Params.from_config(cfg); p.head_dim = 96; p.d_model = 96 * 4
    cases.append((p, -2))
    p = F.Params.from_config(cfg); p.d_model = 200
    cases.append((p, -1))
    p = F.Params.from_config(cfg); p.bits[2] = 3
    cases.append((p, -2))
    p = F.Params.from_config(cfg); p.n_heads = 0
    cases.append((p, -1))
    p = F.Params.from_config(cfg); p.tau = -1.0
    cases.append((p, -1))
    for p, want in cases:
        assert both(p) == (want, want)
