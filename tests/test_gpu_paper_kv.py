"""Parity of the pages' own cache setting on the GPU (INT4 asymmetric groups
of 64 with an fp16 scale and minimum, keys grouped per channel over 64 rows,
values per row over 64 channels, the last 64 tokens in bf16; residuals of
later loops against the previous reconstruction) [FlashLoop App. E
"Quantization setting"; "Looping a Transformer Quadruples the Bill" §3].

Staged: flashloop_paper_kv_quant on the float32 K/V the oracle quantised, its
codes, scales, minima and tail values equal to the oracle's PaperKVStream bit
for bit; the selected-column rebuild and the attention update on the
oracle's streams give the oracle's O within 1e-2.
Chained and free-running end to end as in test_gpu_end_to_end.py."""
import numpy as np
import pytest
import torch

import oracle as O
from workload import CONFIGS, make_hidden_states, make_weights

pytestmark = pytest.mark.gpu

F = pytest.importorskip("cross_loop_sparse_b200.flashloop")
from gpu_helpers import (bf16_rows, bf16_to_torch, f32, row_rel_l2, torch_to_bf16_bits,  # noqa: E402
                         upload_cols, upload_q, upload_sets, upload_state_after)

TOL = 1e-2
CASES = {
    "tiny": lambda: CONFIGS["tiny"],
    "ragged_300": lambda: CONFIGS["tiny"].with_(seq=300),   # a partial key group, tail of 64
    "short_40": lambda: CONFIGS["tiny"].with_(seq=40),      # no body: every token in the bf16 tail
    "ouro14_4k": lambda: CONFIGS["ouro14_4k"],
}
_RUNS = {}


def oracle_run(name):
    if name not in _RUNS:
        cfg = CASES[name]()
        W = make_weights(cfg)
        X, _ = make_hidden_states(cfg)
        _RUNS[name] = (cfg, W, X, O.OracleSequence(cfg, W, X, kv_scheme="paper").run())
    return _RUNS[name]


def pack4(codes):
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack4(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2], out[..., 1::2] = p & 15, p >> 4
    return out


def stream_rows(stream, r):
    """Loop r's quantised rows of an oracle stream in the GPU layout: codes
    [n, H, dh], scales and minima (keys [groups, H, dh], values [n, H, dh/64])."""
    codes, s16, lo16, n = stream.base if r == 1 else stream.res[r]
    if stream.kind == "v":
        return codes.reshape(n, stream.H, stream.dh), s16, lo16
    return codes.transpose(0, 3, 1, 2).reshape(-1, stream.H, stream.dh)[:n], s16, lo16


def gpu_rows(st, name, r, n, ng):
    codes = unpack4(st[f"p{name}_codes{r}"][:n].cpu().numpy())
    s = st[f"p{name}_scale{r}"][:ng].cpu().numpy()
    lo = st[f"p{name}_min{r}"][:ng].cpu().numpy()
    return codes, s, lo


def upload_paper(stream, st, name, r, heads):
    """Write loop r of an oracle stream over the held heads of the GPU's."""
    codes, s16, lo16 = stream_rows(stream, r)
    n, ng = codes.shape[0], s16.shape[0]
    if n:
        st[f"p{name}_codes{r}"][:n, heads] = torch.from_numpy(pack4(codes)).cuda()
        st[f"p{name}_scale{r}"][:ng, heads] = torch.from_numpy(s16).cuda()
        st[f"p{name}_min{r}"][:ng, heads] = torch.from_numpy(lo16).cuda()
    toks, bits = stream.tail_vals[r]
    if toks.size:
        tail = st[f"p{name}_tail{r}"]
        idx = torch.from_numpy(toks - stream.body).cuda()
        sub = tail[idx]
        sub[:, heads] = bf16_to_torch(bits)
        tail[idx] = sub


@pytest.mark.parametrize("name", list(CASES))
def test_paper_quant_bit_exact_on_identical_inputs(name):
    cfg, W, X, orc = oracle_run(name)
    S, H, dh = cfg.seq, cfg.n_heads, cfg.head_dim
    p = F.Params.from_config(cfg, kv_scheme="paper")
    st = F.FlashLoopState(p)
    upload_sets(orc, st, cfg.n_loops)
    ref = {n: O.PaperKVStream(S, H, dh, n) for n in ("k", "v")}
    for r in range(1, cfg.n_loops + 1):
        act = orc.active[r]
        k32 = orc.k_exact[r].astype(np.float32)
        v32 = orc.v_exact[r].astype(np.float32)
        if r == 1:
            F.flashloop_paper_kv_quant(p, 1, f32(k32), f32(v32), None, None, st)
            ref["k"].write_base(k32)
            ref["v"].write_base(v32)
        else:
            F.flashloop_paper_kv_quant(p, r, f32(k32), f32(v32), st[f"active{r}"], st["n_active"][r - 1:], st)
            ref["k"].write_residual(r, act, k32)
            ref["v"].write_residual(r, act, v32)
        torch.cuda.synchronize()
        for n_, stream in ref.items():
            codes, s16, lo16 = stream_rows(stream, r)
            gc, gs, glo = gpu_rows(st, n_, r, codes.shape[0], s16.shape[0])
            assert np.array_equal(gc, codes), (n_, r)
            assert np.array_equal(gs.view(np.uint16), s16.view(np.uint16)), (n_, r)
            assert np.array_equal(glo.view(np.uint16), lo16.view(np.uint16)), (n_, r)
            toks, bits = stream.tail_vals[r]
            gt = torch_to_bf16_bits(st[f"p{n_}_tail{r}"])[toks - stream.body]
            assert np.array_equal(gt, bits), (n_, r)
    assert st.error_code() == 0


@pytest.mark.parametrize("name", ["tiny", "ragged_300", "short_40", "ouro14_4k"])
def test_paper_attention_update_staged(name):
    """Loop by loop on the oracle's streams, sets, queries, selections and
    previous state: the rebuild of the selected columns from the pages'
    streams and the attention update give the oracle's O within 1e-2."""
    cfg, W, X, orc = oracle_run(name)
    p = F.Params.from_config(cfg, kv_scheme="paper")
    st = F.FlashLoopState(p)
    heads = list(range(cfg.n_heads))
    upload_sets(orc, st, cfg.n_loops)
    for r in range(1, cfg.n_loops + 1):
        for n_, stream in (("k", orc.Kc), ("v", orc.Vc)):
            upload_paper(stream, st, n_, r, heads)
        if r > 1:
            upload_state_after(orc, st, r - 1)
            upload_q(orc, st, r - 1)
            upload_cols(orc, st, r)
        upload_q(orc, st, r)
        F.flashloop_selcol_dequant(p, r, st)
        F.flashloop_sparse_attn_update(p, r, st, 1 if r == 1 else 0)
        torch.cuda.synchronize()
        act = orc.active[r]
        err = row_rel_l2(bf16_rows(torch_to_bf16_bits(st["O"])[act]), bf16_rows(orc.O_hist[r][act]))
        assert err.max(initial=0.0) < TOL, (r, float(err.max()))
    assert st.error_code() == 0


def force_paper(cfg, orc, st, r, heads, kx, vx):
    """Loop r's streams: the GPU's equal the oracle's except where the float32
    tensor-core projection and the float64 oracle projection fall on two
    sides of a rounding boundary (a code then differs by one step, a scale or
    minimum by its fp16 spacing plus 1e-5 of the head's largest value, a tail
    value by one bf16 step plus the same); the oracle's are then written over
    the held heads (oracle -> GPU)."""
    for n_, stream, x in (("k", orc.Kc, kx), ("v", orc.Vc, vx)):
        codes, s16, lo16 = stream_rows(stream, r)
        n, ng = codes.shape[0], s16.shape[0]
        gc, gs, glo = gpu_rows(st, n_, r, n, ng)
        gc, gs, glo = gc[:, heads], gs[:, heads], glo[:, heads]
        if n:
            assert np.mean(gc != codes) < 2e-3, (n_, r, float(np.mean(gc != codes)))
            assert np.max(np.abs(gc.astype(np.int32) - codes)) <= 1, (n_, r)
            hmax = np.abs(x).max(axis=(0, 2))[None, :, None]            # per held head
            for got, want in ((gs, s16), (glo, lo16)):
                d = np.abs(got.astype(np.float64) - want.astype(np.float64))
                bound = np.spacing(np.abs(want)).astype(np.float64) + 1e-5 * hmax
                assert np.all(d <= bound), (n_, r, float((d - bound).max()))
        toks, bits = stream.tail_vals[r]
        if toks.size:
            gt = bf16_rows(torch_to_bf16_bits(st[f"p{n_}_tail{r}"])[toks - stream.body][:, heads])
            want = bf16_rows(bits)
            hmax = np.abs(x).max(axis=(0, 2))[None, :, None]
            # one bf16 step of the value, plus the projections' difference
            # (which decides the rounding of values near zero)
            bound = 2.0 ** -7 * np.abs(want) + 1e-5 * hmax
            assert np.all(np.abs(gt - want) <= bound), (n_, r, float((np.abs(gt - want) - bound).max()))
        upload_paper(stream, st, n_, r, heads)


def run_chained_paper(cfg, W, X, orc, heads, check_y):
    """Loops 1..R through the calls flashloop_loop_step makes in the pages'
    setting (gate, gathered projection, asymmetric quantiser, top-k, rebuild,
    attention update, output projection), the oracle's streams and
    selections written over the GPU's after each is checked; O of the held
    heads (and Y with every head held) within TOL on every active row."""
    from test_gpu_end_to_end import force_selection, held_cols
    p = F.Params.from_config(cfg, kv_scheme="paper")
    st = F.FlashLoopState(p)
    S, d = cfg.seq, cfg.d_model
    xs = [bf16_to_torch(x) for x in X]
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    kf = torch.zeros((S, d), dtype=torch.float32, device="cuda")
    vf = torch.zeros_like(kf)
    cols = held_cols(cfg, heads)
    R = cfg.n_loops
    worst = {}
    for r in range(1, R + 1):
        cap = p.capacity[r - 1]
        q_out = st[f"q{st.q_slot(r)}"]
        if r == 1:
            act_t = n_t = None
            F.flashloop_qkv_gathered(p, xs[0], None, None, S, wqkv, st["rope_cs"], q_out, kf, vf)
            F.flashloop_paper_kv_quant(p, 1, kf, vf, None, None, st)
        else:
            prev = None if r == 2 else st[f"active{r - 1}"]
            nprev = None if r == 2 else st["n_active"][r - 2:]
            act_t, n_t = st[f"active{r}"], st["n_active"][r - 1:]
            F.flashloop_gate(p, xs[r - 1], xs[r - 2], prev, nprev, p.capacity[r - 2], act_t, st[f"slot{r}"],
                             n_t, cap, st["workspace"], st["err"])
            F.flashloop_qkv_gathered(p, xs[r - 1], act_t, n_t, cap, wqkv, st["rope_cs"], q_out, kf, vf)
            F.flashloop_paper_kv_quant(p, r, kf, vf, act_t, n_t, st)
        torch.cuda.synchronize()
        act = orc.active[r]
        if r >= 2:
            assert int(st["n_active"][r - 1].item()) == act.size
            assert np.array_equal(st[f"active{r}"][: act.size].cpu().numpy(), act)
        force_paper(cfg, orc, st, r, heads, orc.k_exact[r], orc.v_exact[r])
        if r >= 2 and F.flashloop_selection_loop(p, r) == r:
            k = p.topk[r - 1]
            if r == 2:
                F.flashloop_topk_columns(p, st["colmass0"], None, 0, k, st[f"cols{r}"])
            else:
                ps = F.flashloop_selection_loop(p, r - 1)
                F.flashloop_topk_columns(p, st["colmass1"], st[f"cols{ps}"], p.topk[ps - 1], k, st[f"cols{r}"])
            torch.cuda.synchronize()
            force_selection(p, orc, st, r, heads)
        want_cm = 1 if r == 1 else int(r < R and p.topk[r] < p.topk[r - 1])
        F.flashloop_selcol_dequant(p, r, st)
        F.flashloop_sparse_attn_update(p, r, st, want_cm)
        F.flashloop_out_proj(p, st["O"], act_t, n_t, cap, wo, st["Y"])
        torch.cuda.synchronize()
        og = bf16_rows(torch_to_bf16_bits(st["O"])[act][:, cols])
        e = row_rel_l2(og, bf16_rows(orc.O_hist[r][act]))
        worst[f"O{r}"] = round(float(e.max(initial=0.0)), 5)
        assert np.all(e < TOL), (r, float(e.max()), int(act[np.argmax(e)]))
        if check_y:
            ey = row_rel_l2(bf16_rows(torch_to_bf16_bits(st["Y"])[act]), bf16_rows(orc.Y_hist[r][act]))
            worst[f"Y{r}"] = round(float(ey.max(initial=0.0)), 5)
            assert np.all(ey < TOL), (r, float(ey.max()), int(act[np.argmax(ey)]))
    assert st.error_code() == 0
    return worst


@pytest.mark.parametrize("name", ["tiny", "ragged_300", "short_40", "ouro14_4k"])
def test_paper_loop_step_matches_oracle(name):
    cfg, W, X, orc = oracle_run(name)
    heads = list(range(cfg.n_heads))
    chained = run_chained_paper(cfg, W, X, orc, heads, True)
    # free-running: flashloop_loop_step alone; the sets are exact, the codes
    # equal the oracle's but for rare one-step flips at rounding boundaries
    p = F.Params.from_config(cfg, kv_scheme="paper")
    st = F.FlashLoopState(p)
    xs = [bf16_to_torch(x) for x in X]
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    free = {}
    for r in range(1, cfg.n_loops + 1):
        F.flashloop_loop_step(p, r, xs[r - 1], xs[r - 2] if r > 1 else None, wqkv, wo, st)
        torch.cuda.synchronize()
        act = orc.active[r]
        if r > 1:
            assert int(st["n_active"][r - 1].item()) == act.size
            assert np.array_equal(st[f"active{r}"][: act.size].cpu().numpy(), act)
        for n_, stream in (("k", orc.Kc), ("v", orc.Vc)):
            codes, s16, _ = stream_rows(stream, r)
            gc = gpu_rows(st, n_, r, codes.shape[0], s16.shape[0])[0]
            if codes.size:
                assert np.mean(gc != codes) < 5e-2, (n_, r, float(np.mean(gc != codes)))
        e = row_rel_l2(bf16_rows(torch_to_bf16_bits(st["O"])[act]), bf16_rows(orc.O_hist[r][act]))
        free[f"O{r}"] = round(float(e.max(initial=0.0)), 5)
    assert st.error_code() == 0
    print(name, "chained", chained, "free-running", free)
