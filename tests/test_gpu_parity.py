"""CUDA path vs the CPU oracle on small layers that span several tiles and end in
ragged tails (index lists bit-exact on conditioned inputs, outputs within the
stated tolerance), plus invariants and edge cases of the method."""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from tests.gpu_util import Layer, ensure_built
from tests.helpers import TOL, band_violations, rel_err, relu_band_ambiguous

import activation_sparse_ffn_predict_b200 as A

pytestmark = pytest.mark.gpu

SHAPES = {
    # full-size tiny fp32 layer (d 512 = 4 fp32 tiles, n 1376 = 43 words)
    "tiny_reglu_f32": S.get("tiny_reglu_f32"),
    # fp16 ReGLU: d 1096 = 4 tiles of 256 + 72; n 3000 = 93 words + 24; r 136 = 17 chunks
    "reglu_f16_ragged": S.get("llama2_7b_reglu").with_(d=1096, n=3000, r=136),
    # fp16 plain ReLU: d 1352, n 2085, r 72
    "relu_f16_ragged": S.get("falcon_40b_relu").with_(d=1352, n=2085, r=72),
    # fp32 ReGLU with ragged everything
    "reglu_f32_ragged": S.get("tiny_reglu_f32").with_(d=516, n=1001, r=68, seed=11),
    # fewer neurons than one mask word
    "relu_f16_tiny_n": S.get("opt175b_relu").with_(d=264, n=20, r=16, frac=0.3),
}

BATCHES = [1, 2, 3, 4, 8, 16, 32]


@pytest.fixture(scope="module", params=list(SHAPES))
def layer(request):
    ensure_built()
    return Layer(SHAPES[request.param], n_tokens=48)


def test_conditioned_inputs_have_unique_decisions(layer):
    h = layer.h
    assert band_violations(h["W1"], h["b1"], h["W2"], h["b2"], layer.X, layer.cfg.tau) == 0


@pytest.mark.parametrize("B", BATCHES)
def test_predict_index_list_bit_exact(layer, B):
    for start in (0, 48 - B):
        rows = slice(start, start + B)
        ref = layer.oracle_idx(rows)
        got, raw, c = layer.predict(rows)
        assert got.dtype == np.int32
        np.testing.assert_array_equal(got, ref)
        # entries past count untouched
        assert np.all(raw[c:] == -7)
    assert layer.error() == 0


@pytest.mark.parametrize("B", BATCHES)
def test_sparse_ffn_matches_oracle(layer, B):
    rows = slice(3, 3 + B)
    idx = layer.oracle_idx(rows)
    ref = layer.oracle_y(rows, idx)
    y = layer.sparse(rows, idx)
    assert np.isfinite(y).all()
    assert rel_err(y, ref) <= TOL[layer.cfg.dtype], rel_err(y, ref)
    assert layer.error() == 0


@pytest.mark.parametrize("B", [1, 4, 32])
def test_predict_then_sparse_end_to_end(layer, B):
    rows = slice(10, 10 + B)
    x = layer.Xd[rows].contiguous()
    n = layer.cfg.n
    idx = torch.zeros(n, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.zeros(B, layer.cfg.d, dtype=torch.float32, device="cuda")
    A.asf_predict(layer.pred, x, layer.cfg.tau, idx, cnt, layer.ws)
    A.asf_sparse_ffn(layer.ffn, x, idx, cnt, y, layer.ws)
    torch.cuda.synchronize()
    ref_idx = layer.oracle_idx(rows)
    assert int(cnt.item()) == ref_idx.size
    ref = layer.oracle_y(rows, ref_idx)
    assert rel_err(y.cpu().numpy(), ref) <= TOL[layer.cfg.dtype]


@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8, 12, 32])
def test_combined_call_is_bitwise_the_two_calls(layer, B):
    # asf_predict_sparse_ffn: for small batches the FFN kernel ranks the union
    # mask itself (no compaction kernel); idx, count and y equal those of
    # asf_predict + asf_sparse_ffn bit for bit, and match the oracle
    rows = slice(5, 5 + B)
    x = layer.Xd[rows].contiguous()
    n, d = layer.cfg.n, layer.cfg.d
    outs = []
    for mode in ("two calls", "combined", "halves"):
        idx = torch.full((n,), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        y = torch.full((B, d), float("nan"), dtype=torch.float32, device="cuda")
        args = (layer.pred, layer.ffn, x, layer.cfg.tau, idx, cnt, y, layer.ws)
        if mode == "combined":
            A.asf_predict_sparse_ffn(*args)
        elif mode == "halves":
            # the combined call in its two halves, split where a caller may put an event
            A.asf_predict_sparse_ffn_begin(*args)
            torch.cuda.current_stream().record_event(torch.cuda.Event())
            A.asf_predict_sparse_ffn_end(*args)
        else:
            A.asf_predict(layer.pred, x, layer.cfg.tau, idx, cnt, layer.ws)
            A.asf_sparse_ffn(layer.ffn, x, idx, cnt, y, layer.ws)
        torch.cuda.synchronize()
        outs.append((idx.cpu().numpy(), int(cnt.item()), y.cpu().numpy()))
    (i0, c0, y0) = outs[0]
    for (i1, c1, y1) in outs[1:]:
        assert c0 == c1
        np.testing.assert_array_equal(i0, i1)          # the list, and the untouched tail
        assert (i1[c1:] == -7).all()
        np.testing.assert_array_equal(y0, y1)
    ref_idx = layer.oracle_idx(rows)
    np.testing.assert_array_equal(i1[:c1], ref_idx)
    assert rel_err(y1, layer.oracle_y(rows, ref_idx)) <= TOL[layer.cfg.dtype]
    assert layer.error() == 0


@pytest.mark.parametrize("B", [1, 5, 32])
def test_dense_matches_oracle(layer, B):
    rows = slice(0, B)
    h = layer.h
    ref = O.dense_ffn(h["act"], h["Wg"], h["Wu"], h["WdT"], h["bias"], layer.X[rows])
    assert rel_err(layer.dense(rows), ref) <= TOL[layer.cfg.dtype]


def test_sparse_over_true_set_equals_dense(layer):
    # Invariant: inactive neurons contribute exactly zero, so the sparse output
    # over T(x) (or any superset) is the dense output up to reassociation.
    h = layer.h
    for t in range(4):
        rows = slice(t, t + 1)
        T = np.flatnonzero(O.true_active(h["act"], h["Wg"], h["Wu"], h["bias"], layer.X[rows])[0])
        yd = layer.dense(rows)
        ys = layer.sparse(rows, T)
        assert rel_err(ys, yd) <= TOL[layer.cfg.dtype]
        sup = np.union1d(T, np.arange(0, layer.cfg.n, 3))
        assert rel_err(layer.sparse(rows, sup), yd) <= TOL[layer.cfg.dtype]


def test_all_neurons_list_is_bitwise_dense(layer):
    rows = slice(0, 3)
    np.testing.assert_array_equal(layer.sparse(rows, np.arange(layer.cfg.n)), layer.dense(rows))


def test_disjoint_and_empty_lists_give_exact_zero(layer):
    h = layer.h
    rows = slice(2, 3)
    act = O.true_active(h["act"], h["Wg"], h["Wu"], h["bias"], layer.X[rows])[0]
    amb = relu_band_ambiguous(h["act"], h["Wg"], h["Wu"], h["bias"], layer.X[rows])[0]
    off = np.flatnonzero(~act & ~amb)
    y = layer.sparse(rows, off)
    assert np.array_equal(y, np.zeros_like(y))
    y0 = layer.sparse(slice(0, 4), [])
    assert np.array_equal(y0, np.zeros_like(y0))
    assert layer.error() == 0


def test_results_are_deterministic(layer):
    rows = slice(0, 4)
    idx = layer.oracle_idx(rows)
    a = layer.sparse(rows, idx)
    b = layer.sparse(rows, idx)
    np.testing.assert_array_equal(a, b)


def test_unsorted_and_duplicate_lists(layer):
    rows = slice(1, 2)
    idx = layer.oracle_idx(rows)
    rng = np.random.default_rng(0)
    shuffled = rng.permutation(idx)
    ref = layer.oracle_y(rows, idx)
    assert rel_err(layer.sparse(rows, shuffled), ref) <= TOL[layer.cfg.dtype]
    if idx.size:
        dup = np.concatenate([idx, idx[:1]])
        assert rel_err(layer.sparse(rows, dup), layer.oracle_y(rows, dup)) <= TOL[layer.cfg.dtype]


def test_out_of_range_index_is_skipped_and_flagged(layer):
    rows = slice(0, 2)
    idx = layer.oracle_idx(rows)
    assert layer.error() == 0
    bad = np.concatenate([idx, np.array([layer.cfg.n, -1, 1 << 30], dtype=np.int64)])
    y = layer.sparse(rows, bad)
    assert layer.error() == A._lib.ASF_ERR_DEVICE_INDEX
    assert layer.error() == 0           # reading clears the word
    assert rel_err(y, layer.oracle_y(rows, idx)) <= TOL[layer.cfg.dtype]


def test_count_above_n_is_clamped_and_flagged(layer):
    rows = slice(0, 1)
    n = layer.cfg.n
    y = layer.sparse(rows, np.arange(n), count=n + 5)
    assert layer.error() == A._lib.ASF_ERR_DEVICE_INDEX
    assert rel_err(y, layer.dense(rows)) <= TOL[layer.cfg.dtype]


# ------------------------------------------------------------- offline path --
def test_activation_counts_within_rounding_band(layer):
    h = layer.h
    cfg = layer.cfg
    Xc = S.layer_tokens(cfg, 0, 300, kind="x_calib")
    Xn = Xc.numpy()
    counts = torch.zeros(cfg.n, dtype=torch.int64, device="cuda")
    A.asf_activation_counts(layer.ffn, Xc[:123].cuda().contiguous(), counts, layer.ws)
    A.asf_activation_counts(layer.ffn, Xc[123:].cuda().contiguous(), counts, layer.ws)
    got = counts.cpu().numpy()
    pre = O.relu_input(h["act"], h["Wg"], h["Wu"], h["bias"], Xn)
    amb = relu_band_ambiguous(h["act"], h["Wg"], h["Wu"], h["bias"], Xn)
    lo = ((pre > 0) & ~amb).sum(axis=0)
    hi = ((pre > 0) | amb).sum(axis=0)
    assert np.all(got >= lo) and np.all(got <= hi)
    exact = O.profile_counts(h["act"], h["Wg"], h["Wu"], h["bias"], Xn)
    assert np.mean(got == exact) > 0.999


def test_hot_permutation_pipeline_preserves_outputs(layer):
    cfg = layer.cfg
    Xc = S.layer_tokens(cfg, 0, 200, kind="x_calib").cuda().contiguous()
    counts = torch.zeros(cfg.n, dtype=torch.int64, device="cuda")
    A.asf_activation_counts(layer.ffn, Xc, counts, layer.ws)
    perm = A.asf_hot_permutation(counts.cpu().numpy())
    np.testing.assert_array_equal(perm, O.hot_permutation(counts.cpu().numpy()))
    perm_d = torch.from_numpy(perm).cuda()
    w = layer.w

    def prow(t):
        if t is None:
            return None
        out = torch.empty_like(t)
        A.asf_permute_rows(t, out, perm_d)
        return out

    pw = {k: prow(getattr(w, k)) for k in ["Wg", "Wu", "WdT", "bias", "W2", "b2"]}
    torch.cuda.synchronize()
    for k, t in pw.items():
        if t is not None:
            assert torch.equal(t.cpu(), getattr(w, k).cpu()[perm.astype(np.int64)])
    pred = A.Predictor(w.W1, w.b1, pw["W2"], pw["b2"])
    ffn = A.FFN(w.act, pw["Wg"], pw["Wu"], pw["WdT"], pw["bias"])
    ws = A.Workspace(pred, ffn, 8)
    rows = slice(0, 4)
    x = layer.Xd[rows].contiguous()
    idx = torch.zeros(cfg.n, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.zeros(4, cfg.d, dtype=torch.float32, device="cuda")
    A.asf_predict(pred, x, cfg.tau, idx, cnt, ws)
    A.asf_sparse_ffn(ffn, x, idx, cnt, y, ws)
    torch.cuda.synchronize()
    got = idx[: int(cnt.item())].cpu().numpy()
    ref_ids = layer.oracle_idx(rows)
    inv = O.inverse_permutation(perm)
    np.testing.assert_array_equal(got, np.sort(inv[ref_ids]))
    assert np.all(np.diff(got) > 0)
    assert rel_err(y.cpu().numpy(), layer.oracle_y(rows, ref_ids)) <= TOL[cfg.dtype]
    # the hot rows come first: counts are non-increasing in storage order
    c_sorted = counts.cpu().numpy()[perm.astype(np.int64)]
    assert np.all(np.diff(c_sorted) <= 0)


def test_permute_rows_unaligned_units():
    ensure_built()
    src = torch.arange(7 * 6, dtype=torch.uint8, device="cuda").reshape(7, 6)
    dst = torch.empty_like(src)
    perm = torch.tensor([6, 0, 5, 1, 4, 2, 3], dtype=torch.int32, device="cuda")
    A.asf_permute_rows(src, dst, perm)
    torch.cuda.synchronize()
    assert torch.equal(dst.cpu(), src.cpu()[perm.cpu().long()])


def test_hot_row_hint_changes_nothing_but_speed(layer):
    cfg = layer.cfg
    w = layer.w
    hinted = A.FFN(w.act, w.Wg, w.Wu, w.WdT, w.bias, hot_rows=cfg.n // 2)
    for B in (1, 3):
        rows = slice(0, B)
        idx = layer.oracle_idx(rows)
        x = layer.Xd[rows].contiguous()
        idt = torch.zeros(cfg.n, dtype=torch.int32, device="cuda")
        if idx.size:
            idt[:idx.size] = torch.from_numpy(idx).cuda()
        cnt = torch.tensor([idx.size], dtype=torch.int32, device="cuda")
        y0 = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
        y1 = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
        A.asf_sparse_ffn(layer.ffn, x, idt, cnt, y0, layer.ws)
        A.asf_sparse_ffn(hinted, x, idt, cnt, y1, layer.ws)
        torch.cuda.synchronize()
        assert torch.equal(y0, y1)
    assert layer.error() == 0


def test_l2_next_hint_changes_nothing_but_speed(layer):
    # The hint makes the call's last kernel prefetch other ranges into L2:
    # results of both FFN paths (fused at B <= 4, two-kernel above) and of a
    # dense call are bit-identical with it, and no device error is raised.
    cfg = layer.cfg
    w = layer.w
    hinted = A.FFN(w.act, w.Wg, w.Wu, w.WdT, w.bias)
    hinted.set_l2_next(w.W1, w.W2)
    odd = torch.empty(4 * 1024 + 48, dtype=torch.uint8, device="cuda")    # not a multiple of 16 bytes long
    for B in (1, 3, 16):
        rows = slice(0, B)
        idx = layer.oracle_idx(rows)
        x = layer.Xd[rows].contiguous()
        idt = torch.zeros(cfg.n, dtype=torch.int32, device="cuda")
        if idx.size:
            idt[:idx.size] = torch.from_numpy(idx).cuda()
        cnt = torch.tensor([idx.size], dtype=torch.int32, device="cuda")
        y0 = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
        y1 = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
        A.asf_sparse_ffn(layer.ffn, x, idt, cnt, y0, layer.ws)
        A.asf_sparse_ffn(hinted, x, idt, cnt, y1, layer.ws)
        torch.cuda.synchronize()
        assert torch.equal(y0, y1)
        hinted.set_l2_next(odd[:4 * 1024 + 40])
        A.asf_dense_ffn(layer.ffn, x, y0, layer.ws)
        A.asf_dense_ffn(hinted, x, y1, layer.ws)
        torch.cuda.synchronize()
        assert torch.equal(y0, y1)
        hinted.set_l2_next(w.W1, w.W2)
    assert layer.error() == 0


def test_packed_layout_is_bitwise_equal_to_split_layout(layer):
    # Neuron-major packed rows (one bulk copy per neuron) change the memory
    # layout only: every FFN path must give bit-identical results.
    cfg = layer.cfg
    w = layer.w
    packed = A.pack_layer(w.act, w.Wg, w.Wu, w.WdT)
    pf = A.FFN.packed(w.act, packed, w.bias, hot_rows=cfg.n // 4)
    for B in (1, 4, 16):
        rows = slice(0, B)
        x = layer.Xd[rows].contiguous()
        ids = layer.oracle_idx(rows)
        idt = torch.zeros(cfg.n, dtype=torch.int32, device="cuda")
        if ids.size:
            idt[:ids.size] = torch.from_numpy(ids).cuda()
        cnt = torch.tensor([ids.size], dtype=torch.int32, device="cuda")
        ys = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
        yp = torch.zeros(B, cfg.d, dtype=torch.float32, device="cuda")
        A.asf_sparse_ffn(layer.ffn, x, idt, cnt, ys, layer.ws)
        A.asf_sparse_ffn(pf, x, idt, cnt, yp, layer.ws)
        torch.cuda.synchronize()
        assert torch.equal(ys, yp), B
        A.asf_dense_ffn(layer.ffn, x, ys, layer.ws)
        A.asf_dense_ffn(pf, x, yp, layer.ws)
        torch.cuda.synchronize()
        assert torch.equal(ys, yp), B
    Xc = S.layer_tokens(cfg, 0, 64, kind="x_calib").cuda().contiguous()
    c1 = torch.zeros(cfg.n, dtype=torch.int64, device="cuda")
    c2 = torch.zeros(cfg.n, dtype=torch.int64, device="cuda")
    A.asf_activation_counts(layer.ffn, Xc, c1, layer.ws)
    A.asf_activation_counts(pf, Xc, c2, layer.ws)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)
    assert layer.error() == 0


def test_gather_rows_strided_and_permuted():
    ensure_built()
    src = torch.arange(9 * 24, dtype=torch.int16, device="cuda").reshape(9, 24)
    perm = torch.tensor([8, 0, 3, 3, 7, 1, 2, 6, 5], dtype=torch.int32, device="cuda")
    dst = torch.full((9, 2, 24), -1, dtype=torch.int16, device="cuda")
    A.asf_gather_rows(src, dst, perm, dst_offset=48, dst_stride=96)
    torch.cuda.synchronize()
    assert torch.equal(dst[:, 1].cpu(), src.cpu()[perm.cpu().long()])
    assert (dst[:, 0] == -1).all()
    with pytest.raises(ValueError):
        A.asf_gather_rows(src, dst, perm, dst_offset=96, dst_stride=96)
