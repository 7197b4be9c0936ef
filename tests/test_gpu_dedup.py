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


def _close(got, ref):
    g, r = _bf16_f64(got), _bf16_f64(ref)
    assert (np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + 1e-3).all()
    assert (got == ref).mean() >= 0.999


CASES = [("tiny", None, 0), ("decode", None, 1), ("skewed", 512, 0), ("prefill", 256, 2)]


@pytest.mark.parametrize("name,T,seed", CASES, ids=[c[0] for c in CASES])
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
    assert np.array_equal(_host(dd["dd_x"][:D]), o_d["recv_x"])
    if w.fp8:
        assert np.array_equal(_host(dd["dd_scale"][:D]).view(np.uint32), o_d["recv_scale"].view(np.uint32))

    # permute -> the standard expert-grouped receive buffers
    pipe.permute()
    assert pipe.check_errors() == 0
    assert np.array_equal(_host(pipe.recv["recv_x"][:M]), o_rx)
    assert np.array_equal(_host(pipe.recv["recv_src"][:M]), o_src)
    if w.fp8:
        assert np.array_equal(_host(pipe.recv["recv_scale"][:M]).view(np.uint32), o_rs.view(np.uint32))

    # local reduce + cross-rank combine
    if w.fp8 and not fused:
        pipe.identity_expert()
    pipe.local_reduce(fused=fused)
    pipe.combine_dedup()
    assert pipe.check_errors() == 0
    _close(_host(dd["partial"][:D]), o_part)
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
