"""Grouped SwiGLU GEMMs (tcgen05) and the whole layer on the GPU against the
oracle: small shapes that span several tiles with ragged tails and empty
experts, then every workload at full size on sampled tokens."""
import contextlib

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import WORKLOADS, adversarial_logits, make_inputs
from tests._util import (assert_close_layer, assert_close_scaled, np64,
                         route_equals_oracle_own_logits, router_logits_checked)

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


@contextlib.contextmanager
def _gemm_form(form):
    """Force the grouped GEMMs' tile form (rows / token columns) inside."""
    moe = _moe()
    code = {"auto": moe.GEMM_FORM_AUTO, "rows": moe.GEMM_FORM_ROWS,
            "tokens": moe.GEMM_FORM_TOKENS}[form]
    moe.moe_debug_set_gemm_form(code)
    try:
        yield
    finally:
        moe.moe_debug_set_gemm_form(moe.GEMM_FORM_AUTO)


def _problem(T, d, F, E, k, dtype, seed, skew=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(dtype)
    s_in, s_mid = d ** -0.5, F ** -0.5
    W1 = (torch.randn(E, F, d, generator=g) * s_in).to(dtype)
    W3 = (torch.randn(E, F, d, generator=g) * s_in).to(dtype)
    W2 = (torch.randn(E, d, F, generator=g) * s_mid).to(dtype)
    lg = adversarial_logits(T, E, "normal", seed=seed).numpy()
    if skew and E >= 4:
        lg[:, 1] -= 40.0   # expert 1 empty
        lg[:, 0] += 3.0    # expert 0 heavy (several tiles)
    return x, W1, W3, W2, lg


def _expert_ref(x, W1, W3, W2, lg, k):
    E = W1.shape[0]
    idx, gate, _ = O.route(lg, k)
    meta = O.routing_metadata(idx, E)
    Xe = O.dispatch(x.double().numpy(), meta["slot"])
    Ye, A, B, H = O.expert_ffn(Xe, meta["offsets"], np64(W1), np64(W3), np64(W2), keep=True)
    return meta, gate, Xe, H, Ye


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,F,E,k", [(300, 256, 256, 5, 2), (129, 128, 384, 3, 1),
                                       (700, 512, 128, 16, 4), (5, 256, 128, 4, 2),
                                       (1000, 384, 256, 7, 3),
                                       # at least 512 rows per expert on average: the
                                       # down GEMM on 256-row CTA-pair tiles (with an
                                       # empty and a heavy expert, ragged tails)
                                       (1500, 256, 256, 2, 2), (2100, 512, 384, 4, 3)])
def test_grouped_swiglu_small(dtype, T, d, F, E, k):
    moe = _moe()
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, dtype, seed=T + d + F)
    meta, gate, Xe_ref, H_ref, Ye_ref = _expert_ref(x, W1, W3, W2, lg, k)
    dev = "cuda"
    Xe = torch.from_numpy(Xe_ref).to(dtype).to(dev)  # exact: Xe rows are rows of x
    offs = torch.from_numpy(meta["offsets"]).to(dev)
    H, Ye = moe.moe_grouped_swiglu(Xe, W1.to(dev), W3.to(dev), W2.to(dev), offs)
    assert moe.moe_get_status() == 0
    assert_close_scaled(np64(H), H_ref, "H")
    assert_close_scaled(np64(Ye), Ye_ref, "Ye")


# expert row counts whose last 128-row tile holds 1, 15, 16, 17, 31, 33, 64,
# 127, 128 (full) or 0 (empty expert) rows, several experts spanning more
# than one tile
TAIL_COUNTS = [1, 15, 16, 17, 31, 33, 127, 128, 129, 200, 0, 255, 257, 64, 384, 3]


# larger experts: after 0, 1 or 2 full 256-row chunks the last rows number
# 1, 64, 127, 128, 129, 200, 255 or 256; an empty expert too
LARGER_COUNTS = [1, 64, 127, 128, 129, 200, 255, 256, 257, 300, 384, 385, 511, 512, 0, 640]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d,F", [(256, 256), (384, 128), (512, 384)])
@pytest.mark.parametrize("which", ["small_experts", "larger_experts"])
@pytest.mark.parametrize("form", ["rows", "tokens"])
def test_grouped_swiglu_every_tail_size(dtype, d, F, which, form):
    """Expert segments given directly by offsets, so every ragged tail size
    is met, with 16 experts averaging 104 rows and with experts averaging
    259 rows, on row tiles (128-row single-CTA tiles; the down GEMM on CTA
    pairs where experts average 512 rows or more) and on token-column tiles
    (256-row chunks and a last chunk of 1 .. 256 rows; d = 384 keeps the
    down GEMM on row tiles); A, B and H kept for the backward are checked
    too."""
    with _gemm_form(form):
        _every_tail_size(dtype, d, F, which)


def _every_tail_size(dtype, d, F, which):
    moe = _moe()
    counts = np.array(TAIL_COUNTS if which == "small_experts" else LARGER_COUNTS,
                      dtype=np.int64)
    E, R = len(counts), int(counts.sum())
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    g = torch.Generator().manual_seed(d + F)
    Xe = torch.randn(R, d, generator=g).to(dtype)
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(dtype)
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(dtype)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(dtype)
    Ye_ref, A_ref, B_ref, H_ref = O.expert_ffn(np64(Xe), offsets, np64(W1), np64(W3), np64(W2),
                                               keep=True)
    dev = "cuda"
    offs = torch.from_numpy(offsets).to(dev)
    nan = lambda n: torch.full((R, n), float("nan"), dtype=dtype, device=dev)
    H, A, B = moe.moe_grouped_gate_up_save(Xe.to(dev), W1.to(dev), W3.to(dev), offs,
                                           H=nan(F), A=nan(F), B=nan(F))
    Ye = moe.moe_grouped_down(H, W2.to(dev), offs, Ye=nan(d))
    assert moe.moe_get_status() == 0
    assert_close_scaled(np64(A), A_ref, "A")
    assert_close_scaled(np64(B), B_ref, "B")
    assert_close_scaled(np64(H), H_ref, "H")
    assert_close_scaled(np64(Ye), Ye_ref, "Ye")
    # every row of every expert was written (a missed row stays NaN)
    for t in (H, A, B, Ye):
        assert torch.isfinite(t.float()).all()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,F,E,k", [(300, 256, 256, 5, 2), (5, 256, 128, 4, 2),
                                       (1000, 384, 256, 7, 3), (129, 128, 384, 3, 1),
                                       (2100, 512, 384, 4, 3)])
def test_gate_up_gather_equals_dispatched(dtype, T, d, F, E, k):
    """The fused path (row_token + A rows gathered from x by TMA) computes
    exactly what the dispatch path does: same rows, same MMA order, so H is
    identical bit for bit; and it matches the oracle."""
    moe = _moe()
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, dtype, seed=3 * T + d)
    idx, gate, _ = O.route(lg, k)
    meta = O.routing_metadata(idx, E)
    dev = "cuda"
    xd, W1d, W3d = x.to(dev), W1.to(dev), W3.to(dev)
    slot = torch.from_numpy(meta["slot"]).to(dev)
    offs = torch.from_numpy(meta["offsets"]).to(dev)
    rt = moe.moe_row_token(slot)
    want_rt = np.empty(T * k, np.int32)
    want_rt[meta["slot"].reshape(-1)] = np.repeat(np.arange(T, dtype=np.int32), k)
    assert np.array_equal(rt.cpu().numpy(), want_rt)
    Hg = moe.moe_grouped_gate_up_gather(xd, rt, W1d, W3d, offs)
    Hd = moe.moe_grouped_gate_up(moe.moe_dispatch(xd, slot), W1d, W3d, offs)
    assert moe.moe_get_status() == 0
    assert torch.equal(Hg, Hd)
    Xe = O.dispatch(x.double().numpy(), meta["slot"])
    _, _, _, H_ref = O.expert_ffn(Xe, meta["offsets"], np64(W1), np64(W3), np64(W2), keep=True)
    assert_close_scaled(np64(Hg), H_ref, "H gathered")


def test_gate_up_gather_flags_bad_token():
    """A row_token outside [0, T) is never used as an address: that row is
    computed from token 0 and the status word says so; the other rows are
    unaffected."""
    moe = _moe()
    T, d, F, E, k = 64, 256, 128, 4, 2
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, torch.bfloat16, seed=11)
    idx, gate, _ = O.route(lg, k)
    meta = O.routing_metadata(idx, E)
    dev = "cuda"
    xd, W1d, W3d = x.to(dev), W1.to(dev), W3.to(dev)
    slot = torch.from_numpy(meta["slot"]).to(dev)
    offs = torch.from_numpy(meta["offsets"]).to(dev)
    rt = moe.moe_row_token(slot)
    good = moe.moe_grouped_gate_up_gather(xd, rt, W1d, W3d, offs)
    bad_rt = rt.clone()
    bad_rt[5] = T + 5
    bad_rt[9] = -1
    H = moe.moe_grouped_gate_up_gather(xd, bad_rt, W1d, W3d, offs)
    assert moe.moe_get_status(clear=True) & moe.MOE_DEVERR_BAD_INDEX
    keep = torch.ones(T * k, dtype=torch.bool, device=dev)
    keep[5] = keep[9] = False
    assert torch.equal(H[keep], good[keep])
    assert moe.moe_get_status() == 0


def test_row_token_flags_bad_slot():
    moe = _moe()
    slot = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda")  # 9 >= R = 4
    rt = torch.full((4,), -7, dtype=torch.int32, device="cuda")
    moe.moe_row_token(slot, rt)
    assert moe.moe_get_status(clear=True) & moe.MOE_DEVERR_BAD_INDEX
    assert rt.cpu().tolist() == [0, 0, 1, -7]
    assert moe.moe_get_status() == 0


def test_grouped_gate_up_fused_gate_up_layout():
    """W1/W3 as the two halves of one [E, 2F, d] gate_up tensor."""
    moe = _moe()
    T, d, F, E, k = 400, 256, 256, 6, 2
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, torch.bfloat16, seed=42)
    meta, gate, Xe_ref, H_ref, Ye_ref = _expert_ref(x, W1, W3, W2, lg, k)
    gate_up = torch.cat([W1, W3], dim=1).cuda()
    Xe = torch.from_numpy(Xe_ref).to(torch.bfloat16).cuda()
    H = moe.moe_grouped_gate_up(Xe, gate_up[:, :F], gate_up[:, F:],
                                torch.from_numpy(meta["offsets"]).cuda())
    assert_close_scaled(np64(H), H_ref, "H")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("counts,form", [(TAIL_COUNTS, "rows"), (TAIL_COUNTS, "tokens"),
                                         (LARGER_COUNTS, "rows"), (LARGER_COUNTS, "tokens"),
                                         ([600, 700, 0, 1300], "rows")])
def test_grouped_down_gated_every_tail_size(dtype, counts, form):
    """The down GEMM with each row's gate applied in the epilogue, on row
    tiles (the last case on CTA-pair row tiles: experts averaging 650 rows)
    and on token-column tiles: Ye[r] = gate[r] * (H[r] W2_e^T)."""
    moe = _moe()
    counts = np.array(counts, dtype=np.int64)
    E, R, d, F = len(counts), int(counts.sum()), 512, 256
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    g = torch.Generator().manual_seed(R)
    H = torch.randn(R, F, generator=g).to(dtype)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(dtype)
    rg = torch.rand(R, generator=g) * 0.9 + 0.05
    ref = np.empty((R, d))
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        ref[a:b] = np64(H[a:b]) @ np64(W2[e]).T
    ref *= rg.double().numpy()[:, None]
    offs = torch.from_numpy(offsets).cuda()
    Ye = torch.full((R, d), float("nan"), dtype=dtype, device="cuda")
    with _gemm_form(form):
        moe.moe_grouped_down_gated(H.cuda(), W2.cuda(), offs, rg.cuda(), Ye=Ye)
        plain = moe.moe_grouped_down(H.cuda(), W2.cuda(), offs)
    assert moe.moe_get_status() == 0
    assert torch.isfinite(Ye.float()).all()
    assert_close_scaled(np64(Ye), ref, "Ye")
    # the gate multiplies the fp32 sum once: within one rounding of the
    # ungated row times the gate
    unit = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -23
    scaled = np64(plain) * rg.double().numpy()[:, None]
    assert np.all(np.abs(np64(Ye) - scaled) <= 2.5 * unit * np.abs(scaled) + 1e-30)


@pytest.mark.parametrize("form", ["rows", "tokens"])
def test_layer_fwd_gates_in_down_epilogue(form):
    """moe_layer_fwd without kept rows applies the gates in the down GEMM's
    epilogue; with them (save) the combine applies them. Both match the
    oracle, and the routing is the same."""
    moe = _moe()
    T, d, F, E, k = 1100, 256, 256, 4, 2
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, torch.bfloat16, seed=46)
    ref = O.moe_layer(x, k, W1, W3, W2, logits=lg)
    with _gemm_form(form):
        args = (x.cuda(), k, W1.cuda(), W3.cuda(), W2.cuda())
        gated = moe.moe_layer_fwd(*args, logits=torch.from_numpy(lg).cuda())
        kept = moe.moe_layer_fwd(*args, logits=torch.from_numpy(lg).cuda(), save=True)
    assert moe.moe_get_status() == 0
    assert torch.equal(gated.idx, kept.idx) and torch.equal(gated.slot, kept.slot)
    assert_close_layer(np64(gated.out), ref["out"], "out (gated)")
    assert_close_layer(np64(kept.out), ref["out"], "out (kept)")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_token_tiles_equal_row_tiles_bitwise(dtype):
    """Both tile forms sum each output over K in the same order, so H, the
    saved pre-activations and Ye agree bit for bit."""
    moe = _moe()
    counts = np.array(LARGER_COUNTS + TAIL_COUNTS, dtype=np.int64)
    E, R, d, F = len(counts), int(counts.sum()), 512, 256
    offs = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).cuda()
    g = torch.Generator().manual_seed(5)
    Xe = torch.randn(R, d, generator=g).to(dtype).cuda()
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(dtype).cuda()
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(dtype).cuda()
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(dtype).cuda()
    out = {}
    for form in ("rows", "tokens"):
        with _gemm_form(form):
            H, A, B = moe.moe_grouped_gate_up_save(Xe, W1, W3, offs)
            Ye = moe.moe_grouped_down(H, W2, offs)
        out[form] = (H, A, B, Ye)
    assert moe.moe_get_status() == 0
    for a, b, name in zip(out["rows"], out["tokens"], "H A B Ye".split()):
        assert torch.equal(a, b), name


@pytest.mark.parametrize("w3_first", [False, True])
def test_token_tiles_fused_gate_up_either_order(w3_first):
    """Token-column gate/up on the two halves of one [E, 2F, d] tensor, W1
    the first half or the second (the map then starts at W3 and the
    epilogue takes the gate from the upper lanes)."""
    moe = _moe()
    T, d, F, E, k = 900, 256, 256, 3, 2
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, torch.bfloat16, seed=43)
    meta, gate, Xe_ref, H_ref, Ye_ref = _expert_ref(x, W1, W3, W2, lg, k)
    both = torch.cat([W3, W1] if w3_first else [W1, W3], dim=1).cuda()
    w1 = both[:, F:] if w3_first else both[:, :F]
    w3 = both[:, :F] if w3_first else both[:, F:]
    Xe = torch.from_numpy(Xe_ref).to(torch.bfloat16).cuda()
    offs = torch.from_numpy(meta["offsets"]).cuda()
    with _gemm_form("tokens"):
        H, A, B = moe.moe_grouped_gate_up_save(Xe, w1, w3, offs)
    assert moe.moe_get_status() == 0
    assert_close_scaled(np64(H), H_ref, "H")
    with _gemm_form("rows"):
        H2, A2, B2 = moe.moe_grouped_gate_up_save(Xe, w1, w3, offs)
    assert torch.equal(H, H2) and torch.equal(A, A2) and torch.equal(B, B2)


def test_token_form_falls_back_on_padded_expert_stride():
    """An expert stride that is not a whole number of 16-row groups (gate/up)
    or of rows (down) cannot be mapped for token columns: the row tiles run
    instead, with the same results."""
    moe = _moe()
    T, d, F, E, k = 700, 256, 256, 4, 2
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, torch.bfloat16, seed=44)
    meta, gate, Xe_ref, H_ref, Ye_ref = _expert_ref(x, W1, W3, W2, lg, k)
    pad13 = torch.zeros(E, F + 8, d, dtype=torch.bfloat16)
    pad13[:, :F] = W1
    w1 = pad13.cuda()[:, :F]
    pad3 = torch.zeros(E, F + 8, d, dtype=torch.bfloat16)
    pad3[:, :F] = W3
    w3 = pad3.cuda()[:, :F]
    pad2 = torch.zeros(E, d + 1, F, dtype=torch.bfloat16)
    pad2[:, :d] = W2
    w2 = pad2.cuda()[:, :d]
    Xe = torch.from_numpy(Xe_ref).to(torch.bfloat16).cuda()
    offs = torch.from_numpy(meta["offsets"]).cuda()
    with _gemm_form("tokens"):
        H = moe.moe_grouped_gate_up(Xe, w1, w3, offs)
        Ye = moe.moe_grouped_down(H, w2, offs)
    assert moe.moe_get_status() == 0
    assert_close_scaled(np64(H), H_ref, "H")
    assert_close_scaled(np64(Ye), Ye_ref, "Ye")


@pytest.mark.parametrize("form", ["rows", "tokens"])
def test_layer_fwd_save_either_tile_form(form):
    """The whole layer forward (saving A, B and H for the backward) on each
    tile form."""
    moe = _moe()
    T, d, F, E, k = 1500, 256, 256, 4, 2
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, torch.bfloat16, seed=45)
    ref = O.moe_layer(x, k, W1, W3, W2, logits=lg)
    with _gemm_form(form):
        r = moe.moe_layer_fwd(x.cuda(), k, W1.cuda(), W3.cuda(), W2.cuda(),
                              logits=torch.from_numpy(lg).cuda(), save=True)
    assert moe.moe_get_status() == 0
    assert np.array_equal(r.idx.cpu().numpy(), ref["idx"])
    assert_close_layer(np64(r.out), ref["out"], "out")


def test_grouped_gemm_deterministic():
    moe = _moe()
    T, d, F, E, k = 600, 512, 256, 8, 2
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, torch.bfloat16, seed=7)
    idx, gate, _ = O.route(lg, k)
    meta = O.routing_metadata(idx, E)
    Xe = moe.moe_dispatch(x.cuda(), torch.from_numpy(meta["slot"]).cuda())
    offs = torch.from_numpy(meta["offsets"]).cuda()
    a = moe.moe_grouped_swiglu(Xe, W1.cuda(), W3.cuda(), W2.cuda(), offs)
    b = moe.moe_grouped_swiglu(Xe, W1.cuda(), W3.cuda(), W2.cuda(), offs)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_bad_offsets_flagged_not_faulted():
    moe = _moe()
    d, F, E = 128, 128, 4
    Xe = torch.zeros(256, d, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(E, F, d, dtype=torch.bfloat16, device="cuda")
    W2 = torch.zeros(E, d, F, dtype=torch.bfloat16, device="cuda")
    offs = torch.tensor([0, 100, 50, 200, 256], dtype=torch.int32, device="cuda")  # not monotone
    H = torch.full((256, F), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_grouped_gate_up(Xe, W, W, offs, H=H)
    st = moe.moe_get_status(clear=True)
    assert st & moe.MOE_DEVERR_BAD_OFFSETS
    assert (H == 7.0).all()  # nothing written
    assert moe.moe_get_status() == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_layer_small_full_check(dtype):
    moe = _moe()
    T, d, F, E, k = 777, 256, 384, 12, 3
    x, W1, W3, W2, lg = _problem(T, d, F, E, k, dtype, seed=99)
    Wr = (torch.randn(E, d, generator=torch.Generator().manual_seed(5)) * 0.05).to(dtype)
    r = moe.moe_layer_fwd(x.cuda(), k, W1.cuda(), W3.cuda(), W2.cuda(), Wr=Wr.cuda(), save=True)
    lg = router_logits_checked(r.logits.cpu().numpy(), x, Wr)
    route_equals_oracle_own_logits(r, x, Wr, k, E)
    ref = O.moe_layer(x, k, W1, W3, W2, logits=lg)
    assert np.array_equal(r.idx.cpu().numpy(), ref["idx"])
    assert np.array_equal(r.slot.cpu().numpy(), ref["slot"])
    assert np.array_equal(r.offsets.cpu().numpy(), ref["offsets"])
    assert_close_layer(np64(r.out), ref["out"], "out")
    assert moe.moe_get_status() == 0


def test_layer_tiny_fp32_workload_full():
    moe = _moe()
    w = WORKLOADS["tiny_fp32"]
    inp = make_inputs(w, "cpu")
    dev = {k_: v.cuda() for k_, v in inp.items()}
    r = moe.moe_layer_fwd(dev["x"], w.k, dev["W1"], dev["W3"], dev["W2"], Wr=dev["Wr"])
    ref = O.moe_layer(inp["x"], w.k, inp["W1"], inp["W3"], inp["W2"], Wr=inp["Wr"])
    assert np.array_equal(r.idx.cpu().numpy(), ref["idx"])
    assert np.array_equal(r.counts.cpu().numpy(), ref["counts"])
    assert_close_layer(np64(r.out), ref["out"], "out")


@pytest.mark.slow
@pytest.mark.parametrize("name", ["olmoe_1b7b", "sweep_e8", "sweep_e32", "sweep_e128",
                                  "sweep_e128_zipf", "fine_grained_e384"])
def test_layer_full_size_sampled(name):
    """Full-size workload in the launch configuration the benchmark times;
    routing checked in full, the output on 64 sampled tokens."""
    moe = _moe()
    w = WORKLOADS[name]
    inp = make_inputs(w, "cuda")
    router = w.logits == "router"
    kw = dict(Wr=inp["Wr"]) if router else dict(logits=inp["logits"])
    r = moe.moe_layer_fwd(inp["x"], w.k, inp["W1"], inp["W3"], inp["W2"], save=router, **kw)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    x_cpu = inp["x"].cpu()
    lg = (router_logits_checked(r.logits.cpu().numpy(), x_cpu, inp["Wr"].cpu()) if router
          else inp["logits"].cpu().numpy())
    if router:
        route_equals_oracle_own_logits(r, x_cpu, inp["Wr"].cpu(), w.k, w.E)
    idx, gate, _ = O.route(lg, w.k)
    meta = O.routing_metadata(idx, w.E)
    assert np.array_equal(r.idx.cpu().numpy(), idx)
    assert np.array_equal(r.slot.cpu().numpy(), meta["slot"])
    assert np.array_equal(r.offsets.cpu().numpy(), meta["offsets"])
    rng = np.random.default_rng(0)
    toks = np.sort(rng.choice(w.T, size=64, replace=False))
    toks[0], toks[-1] = 0, w.T - 1
    ref = O.moe_layer_tokens(x_cpu, toks, idx, gate, inp["W1"], inp["W3"], inp["W2"])
    got = np64(r.out[torch.as_tensor(toks, device="cuda")])
    assert_close_layer(got, ref, name)
