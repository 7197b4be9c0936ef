"""GPU parity of the deduplicated (per destination rank) receive against
the CPU oracle.

Compared bit-exactly:
- the dedup layout (tok_row, rank_row_off, rank_src_off) and the standard
  layout beside it;
- dedup rows (bytes, source ids, localised top-k ids);
- the permuted expert rows, which must equal the standard expert-grouped
  dispatch.

Compared within the parity tolerances:
- localised weights: 2^-22 relative;
- partials and the combined output: |err| <= 2^-7 |ref| + 1e-3, with at
  least 99.9% of elements bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from combine_top_group_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from combine_top_group_b200 import ep, runner
    return ep, runner


def _host(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def _bf16_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def _close(got, ref, chunk=8192):
    """Every element within the tolerance and >= 99.9% bit-exact, compared in
    row chunks (full-size arrays would not fit as fp64)."""
    exact = 0
    for a in range(0, got.shape[0], chunk):
        gb, rb = got[a:a + chunk], ref[a:a + chunk]
        g, r = _bf16_f64(gb), _bf16_f64(rb)
        assert (np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + 1e-3).all(), f"rows {a}.."
        exact += int((gb == rb).sum())
    assert exact >= 0.999 * got.size


def _equal_rows(dev, ref, what, chunk=32768):
    """dev (device rows) equals ref (host rows) bit for bit, copied back in
    chunks."""
    assert dev.shape[0] == ref.shape[0]
    for a in range(0, ref.shape[0], chunk):
        got = _host(dev[a:a + chunk])
        exp = ref[a:a + chunk]
        if got.dtype == np.float32:
            got, exp = got.view(np.uint32), exp.view(np.uint32)
        assert np.array_equal(got, exp), f"{what}: rows {a}.."


# prefill at T = 4096 is the full-size workload: D = 129 866 dedup rows, M = 262 144 expert rows
CASES = [("tiny", None, 0), ("decode", None, 1), ("skewed", 512, 0), ("prefill", 256, 2), ("prefill", None, 1)]


@pytest.mark.parametrize("name,T,seed", CASES, ids=[f"{c[0]}-{c[1] or 'full'}" for c in CASES])
@pytest.mark.parametrize("fused", [False, True], ids=["y_bf16", "y_fused"])
def test_dedup_path_parity(cuda, name, T, seed, fused):
    ep, runner = cuda
    w = wl.WORKLOADS[name]
    if T:
        w = w.with_tokens(T)
    if fused and not w.fp8:
        pytest.skip("fused dequant applies to FP8 rows only")
    x, logits = wl.make_x(w, seed), wl.make_logits(w, seed)
    pipe = runner.Pipeline(w, seed, x=x, logits=logits, dedup=True)

    # oracle
    o_idx, o_w, _ = oracle.route(logits, w.K, w.route, w.G, w.KG)
    if w.mask_frac:
        oracle.apply_mask(o_idx, o_w, w.mask_seed, w.mask_frac)
    o_lay = oracle.layout(o_idx, w.R, w.T, w.E)
    M = int(o_lay["expert_off"][-1])
    o_dd = oracle.layout_dedup(o_lay["is_token_in_rank"], w.R, w.T)
    D = o_dd["D"]
    o_d = oracle.dispatch_dedup(x, o_dd["tok_row"], o_idx, o_w, D, w.E, w.fp8)
    o_rx, o_rs, o_src, o_rw = oracle.permute(o_d, o_lay["dst_row"], M, w.fp8)
    if w.fp8 and not fused:
        y, ys = oracle.identity_expert_fp8(o_rx, o_rs), None
    else:
        y, ys = o_rx, o_rs
    o_part = oracle.local_reduce(y, ys, o_d, o_lay["dst_row"])
    o_out = oracle.combine_dedup(o_part, o_dd["tok_row"])

    # GPU: layout
    pipe.layout()
    assert pipe.check_errors() == 0
    lay = {k: _host(v) for k, v in ep.ep_buffer_layout(pipe.buf, w.T).items()}
    assert np.array_equal(lay["topk_idx"], o_idx)
    for key in ("dst_row", "expert_off", "cnt", "num_tokens_per_rank"):
        assert np.array_equal(lay[key], o_lay[key]), key
    dd = pipe.dd
    assert np.array_equal(_host(dd["tok_row"]), o_dd["tok_row"])
    assert np.array_equal(_host(dd["rank_row_off"]), o_dd["rank_row_off"])
    assert np.array_equal(_host(dd["rank_src_off"]), o_dd["rank_src_off"])
    assert pipe.dedup_rows() == D <= M

    # dispatch_dedup
    pipe.dispatch_dedup()
    assert pipe.check_errors() == 0
    assert np.array_equal(_host(dd["dd_src"][:D]), o_d["recv_src"])
    assert np.array_equal(_host(dd["dd_topk_idx"][:D]), o_d["recv_topk_idx"])
    gw, ow = _host(dd["dd_topk_w"][:D]).astype(np.float64), o_d["recv_topk_w"]
    assert (np.abs(gw - ow) <= 2.0 ** -22 * np.abs(ow)).all()
    _equal_rows(dd["dd_x"][:D], o_d["recv_x"], "dedup rows")
    if w.fp8:
        _equal_rows(dd["dd_scale"][:D], o_d["recv_scale"], "dedup scales")

    # permute -> the standard expert-grouped receive buffers
    pipe.permute()
    assert pipe.check_errors() == 0
    _equal_rows(pipe.recv["recv_x"][:M], o_rx, "expert rows")
    assert np.array_equal(_host(pipe.recv["recv_src"][:M]), o_src)
    if w.fp8:
        _equal_rows(pipe.recv["recv_scale"][:M], o_rs, "expert scales")

    # local reduce + cross-rank combine
    if w.fp8 and not fused:
        pipe.identity_expert()
    pipe.local_reduce(fused=fused)
    pipe.combine_dedup()
    assert pipe.check_errors() == 0
    _close(_host(dd["partial"][:D]), o_part)
    del o_rx, o_d
    _close(_host(pipe.out), o_out)


def test_dedup_calls_need_the_flag(cuda):
    ep, runner = cuda
    w = wl.WORKLOADS["tiny"]
    pipe = runner.Pipeline(w, 0)
    pipe.layout()
    for call in (lambda: ep.ep_dispatch_dedup(pipe.buf, w.T, pipe.x), lambda: ep.ep_permute(pipe.buf, w.T),
                 lambda: ep.ep_combine_dedup(pipe.buf, w.T, pipe.out), lambda: ep.ep_buffer_dedup(pipe.buf, w.T)):
        with pytest.raises(ep.EpError) as ei:
            call()
        assert ei.value.status == ep.EP_ERR_INVALID


@pytest.mark.parametrize("num_sms", [1, 20])
def test_dedup_path_under_sm_budget(cuda, num_sms):
    """Every dedup stage under a num_sms cap (one CTA per SM, looping over
    tokens) gives the uncapped run's bytes: dedup rows, expert rows, partials
    and output; bf16 and FP8 rows, the fused dequant included."""
    ep, runner = cuda
    for name, fused in (("tiny", False), ("decode", True), ("skewed", False)):
        w = wl.WORKLOADS[name]
        if name == "skewed":
            w = w.with_tokens(64)
        pipe = runner.Pipeline(w, 3, dedup=True)
        dd = pipe.dd

        def run():
            pipe.layout()
            pipe.dispatch_dedup()
            pipe.permute()
            if w.fp8 and not fused:
                pipe.identity_expert()
            pipe.local_reduce(fused=fused)
            pipe.combine_dedup()
            assert pipe.check_errors() == 0
            D, M = pipe.dedup_rows(), pipe.num_rows()
            return [t.clone() for t in (dd["dd_x"][:D], pipe.recv["recv_x"][:M], dd["partial"][:D], pipe.out)]

        ref = run()
        ep.ep_buffer_set_num_sms(pipe.buf, num_sms)
        for t in (dd["dd_x"], pipe.recv["recv_x"], dd["partial"], pipe.out):
            t.zero_()
        got = run()
        for a, b in zip(got, ref):
            assert torch.equal(a.view(torch.int8), b.view(torch.int8))
