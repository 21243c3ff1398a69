"""Helpers of the GPU parity tests: moving seeded inputs and oracle stage
inputs to the device (the data always flows oracle/generator -> GPU), and
the comparison metrics."""
import numpy as np
import torch

import oracle as O
from cross_loop_sparse_b200 import flashloop as F


def bf16_to_torch(bits, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(torch.bfloat16).to(device)


def torch_to_bf16_bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def i32(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def f32(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def f16(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float16)).to(device)


def row_rel_l2(got, want):
    """Per-row ||got - want|| / ||want|| (float64)."""
    g = np.asarray(got, dtype=np.float64)
    w = np.asarray(want, dtype=np.float64)
    num = np.linalg.norm(g - w, axis=-1)
    den = np.linalg.norm(w, axis=-1)
    return num / np.maximum(den, 1e-30)


def bf16_rows(bits):
    return O.flashloop_oracle.bf16_vals(bits)


def upload_cache(orc, st, upto):
    """Copy the oracle's packed K/V streams (loops 1..upto) into the GPU state."""
    cfg = orc.cfg
    for name, kv in (("k", orc.Kc), ("v", orc.Vc)):
        codes, s16 = kv.base
        st[f"{name}_base"].copy_(torch.from_numpy(codes.astype(np.int8)))
        st[f"{name}_base_s"].copy_(torch.from_numpy(s16))
        for r in range(2, upto + 1):
            codes, s16 = kv.res[r]
            packed = O.pack_codes(codes, cfg.bits[r - 1])
            n = packed.shape[0]
            st[f"{name}_res{r}"][:n].copy_(torch.from_numpy(packed))
            st[f"{name}_res{r}_s"][:n].copy_(torch.from_numpy(s16))


def upload_sets(orc, st, upto):
    """Active lists, slot maps and counts of loops 2..upto."""
    counts = np.zeros(F.MAX_LOOPS, np.int32)
    counts[0] = orc.S
    for r in range(2, upto + 1):
        act = orc.active[r]
        st[f"active{r}"][: act.size].copy_(torch.from_numpy(act.astype(np.int32)))
        slot = np.full(orc.S, -1, np.int32)
        slot[act] = np.arange(act.size)
        st[f"slot{r}"].copy_(torch.from_numpy(slot))
        counts[r - 1] = act.size
    st["n_active"].copy_(torch.from_numpy(counts))


def upload_state_after(orc, st, r):
    """(m, Z, N) of the oracle after loop r into the GPU slot of loop r."""
    m, Z, N = orc.hist[r]
    i = st.q_slot(r)
    st[f"m{i}"].copy_(torch.from_numpy(m.astype(np.float32)))
    st[f"Z{i}"].copy_(torch.from_numpy(Z.astype(np.float32)))
    st[f"N{i}"].copy_(torch.from_numpy(N.astype(np.float32)))


def upload_q(orc, st, r):
    S, Hs, dh = orc.q[r].shape
    st[f"q{st.q_slot(r)}"].copy_(bf16_to_torch(orc.q[r].reshape(S, Hs * dh)))


def upload_cols(orc, st, r):
    sel = F.flashloop_selection_loop(st.params, r)
    T = np.stack([np.asarray(t) for t in orc.T[sel]]).astype(np.int32)
    st[f"cols{sel}"].copy_(torch.from_numpy(T))
