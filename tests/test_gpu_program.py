"""The one-launch program (mmf_program_init / mmf_program_run) against the single-projection
entry points (bit for bit: same kernels' arithmetic, exact int32 split sums) and against the
oracle (within the output tolerance)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_lm_b200 as mmf
from gpu_helpers import DEV, assert_out_close, oracle_forward_from_parts, to_dev

pytestmark = pytest.mark.gpu


def _block(H, I, T, seed, layers=1, chain=False, x_dtype=np.float16, norm=False):
    """Projections of `layers` HGRNBit-shaped blocks.  Level 2l: i, f, g (x_attn), o (x_o),
    gate (x_mlp, GLU); level 2l+1: down (reads gate's output).  With chain=True, layer l+1's
    x_attn is layer l's down output."""
    xs = {s: to_dev(synth.activations(seed, f"prog/{s}", T, H, dtype=x_dtype))
          for s in ("x_attn", "x_o", "x_mlp")}
    ydt = torch.float32 if x_dtype == np.float32 else torch.float16
    projs, host = [], []
    prev_down = None
    for l in range(layers):
        for p in synth.workloads.block(H, I):
            W = synth.weights(seed + l, f"prog/{p.name}", p.N, p.K)
            Wp, beta = mmf.quantize_weights(to_dev(W))
            n_out = p.N // 2 if p.glu else p.N
            y = torch.full((T, n_out), float("nan"), dtype=ydt, device=DEV)
            g = None
            if norm:
                g = to_dev(synth.norm_weight(seed + l, f"prog/{p.name}", p.K, ones=False))
            level = 2 * l + (1 if p.src == "h" else 0)
            if p.src == "h":
                x = next(q["y"] for q in projs[::-1] if q["glu"])
            elif chain and l > 0 and p.src == "x_attn":
                x = prev_down
            else:
                x = xs[p.src]
            projs.append(dict(x=x, norm_w=g, Wp=Wp, beta=beta, y=y, glu=p.glu, level=level))
            host.append((p, Wp, beta))
            if p.src == "h":
                prev_down = y
    return projs, host


def _reference_outputs(projs):
    """Single-projection entry points in level order (the program's inputs are then the
    same bits)."""
    outs = []
    for q in sorted(range(len(projs)), key=lambda i: projs[i]["level"]):
        p = projs[q]
        f = mmf.bitlinear_glu_forward if p["glu"] else mmf.bitlinear_forward
        outs.append((q, f(p["x"], p["Wp"], p["beta"], norm_w=p["norm_w"], out_dtype=p["y"].dtype)))
    torch.cuda.synchronize()
    return dict(outs)


@pytest.mark.parametrize("T", [1, 2, 3, 8, 17, 33, 64])
def test_program_370m_block_matches_single_calls_and_oracle(T):
    projs, host = _block(1024, 2816, T, seed=T)
    prog = mmf.Program(projs, T)
    for rep in range(2):                         # counters are reset between runs
        for p in projs:
            p["y"].fill_(float("nan"))
        prog.run()
        torch.cuda.synchronize()
        assert mmf.mmf_get_device_status() == 0
        ref = _reference_outputs([dict(p, y=torch.empty_like(p["y"])) for p in projs])
        for i, p in enumerate(projs):
            np.testing.assert_array_equal(p["y"].cpu().numpy(), ref[i].cpu().numpy(),
                                          err_msg=f"projection {i} run {rep}")
    # and the oracle, projection by projection, on the same inputs
    for i, ((spec, Wp, beta), p) in enumerate(zip(host, projs)):
        x = p["x"].cpu().numpy()
        y_ref = oracle_forward_from_parts(x, Wp.cpu().numpy(), float(beta.item()), spec.K,
                                          glu=spec.glu)
        assert_out_close(p["y"].double().cpu().numpy(), y_ref)


def _check_against_oracle(projs, host, norm=False):
    """Every projection of a run program against the oracle's projection, each fed the
    program's own fp16/fp32 input (for a chained input, the program's earlier output)."""
    for i, ((spec, Wp, beta), p) in enumerate(zip(host, projs)):
        g = p["norm_w"].cpu().numpy() if norm and p["norm_w"] is not None else None
        y_ref = oracle_forward_from_parts(p["x"].cpu().numpy(), Wp.cpu().numpy(),
                                          float(beta.item()), spec.K, g=g, glu=spec.glu)
        try:
            assert_out_close(p["y"].double().cpu().numpy(), y_ref)
        except AssertionError as e:
            raise AssertionError(f"projection {i} ({spec.name}): {e}") from None


def test_program_two_chained_1p3b_layers():
    """Two 1.3B-shaped layers chained (layer 2's i/f/g read layer 1's down_proj output): four
    dependency levels.  Each projection matches the single-projection entry point bit for bit
    and the oracle within the output tolerance, both fed the program's own inputs."""
    T = 8
    projs, host = _block(2048, 5632, T, seed=3, layers=2, chain=True)
    prog = mmf.Program(projs, T)
    prog.run()
    torch.cuda.synchronize()
    assert mmf.mmf_get_device_status() == 0
    for i, p in enumerate(projs):
        f = mmf.bitlinear_glu_forward if p["glu"] else mmf.bitlinear_forward
        y1 = f(p["x"], p["Wp"], p["beta"], out_dtype=p["y"].dtype)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(p["y"].cpu().numpy(), y1.cpu().numpy(), err_msg=f"proj {i}")
    _check_against_oracle(projs, host)


@pytest.mark.parametrize("T", [1, 8, 16])
def test_program_2p7b_block_against_oracle(T):
    """A 2.7B-shaped block (hidden 2560, GLU half 7040): down_proj's K = 7040 ends in a partial
    512-wide stage.  Run twice; every projection against the oracle."""
    projs, host = _block(2560, 7040, T, seed=27 + T)
    prog = mmf.Program(projs, T)
    for rep in range(2):
        for p in projs:
            p["y"].fill_(float("nan"))
        prog.run()
        torch.cuda.synchronize()
        assert mmf.mmf_get_device_status() == 0
        _check_against_oracle(projs, host)


def test_program_fp32_inputs_with_norm_weights():
    T = 5
    projs, host = _block(1024, 2816, T, seed=9, x_dtype=np.float32, norm=True)
    prog = mmf.Program(projs, T)
    prog.run()
    torch.cuda.synchronize()
    assert mmf.mmf_get_device_status() == 0
    for i, ((spec, Wp, beta), p) in enumerate(zip(host, projs)):
        x = p["x"].cpu().numpy()
        g = p["norm_w"].cpu().numpy()
        y_ref = oracle_forward_from_parts(x, Wp.cpu().numpy(), float(beta.item()), spec.K,
                                          g=g, glu=spec.glu)
        assert_out_close(p["y"].double().cpu().numpy(), y_ref)


@pytest.mark.parametrize("T", [1, 2, 8, 16, 17, 32, 33, 64])
def test_program_short_rows_and_partial_stages(T):
    """Projections whose units have a single stage (K <= 512), a partial last stage (K not a
    multiple of 512) and several levels, at every token-tile size and its boundaries.  With
    16- and 32-token tiles the MMA warps take alternate stages, so a unit of one stage leaves
    one of them without work: its partial must not be added."""
    shapes = [(128, 256, False, 0), (384, 128, False, 0), (512, 384, True, 0),
              (640, 256, False, 1), (1152, 128, False, 1), (896, 512, True, 2)]
    projs, host = [], []
    xs = {}
    for i, (K, N, glu, level) in enumerate(shapes):
        if K not in xs:
            xs[K] = to_dev(synth.activations(T + K, f"short/x{K}", T, K, dtype=np.float16))
        W = synth.weights(40 + i, f"short/{i}", N, K)
        Wp, beta = mmf.quantize_weights(to_dev(W))
        y = torch.full((T, N // 2 if glu else N), float("nan"), dtype=torch.float16, device=DEV)
        projs.append(dict(x=xs[K], norm_w=None, Wp=Wp, beta=beta, y=y, glu=glu, level=level))
        host.append((K, glu, Wp, beta))
    prog = mmf.Program(projs, T)
    for rep in range(2):
        for p in projs:
            p["y"].fill_(float("nan"))
        prog.run()
        torch.cuda.synchronize()
        assert mmf.mmf_get_device_status() == 0
        ref = _reference_outputs([dict(p, y=torch.empty_like(p["y"])) for p in projs])
        for i, p in enumerate(projs):
            np.testing.assert_array_equal(p["y"].cpu().numpy(), ref[i].cpu().numpy(),
                                          err_msg=f"projection {i} run {rep}")
    for (K, glu, Wp, beta), p in zip(host, projs):
        y_ref = oracle_forward_from_parts(p["x"].cpu().numpy(), Wp.cpu().numpy(),
                                          float(beta.item()), K, glu=glu)
        assert_out_close(p["y"].double().cpu().numpy(), y_ref)


def test_program_refuses_a_workspace_whose_plan_was_overwritten():
    """A run whose workspace no longer holds its plan (here the header is zeroed after the
    init) must not touch anything: every CTA returns at once and the status word reports
    MMF_ERR_PLAN.  A fresh init makes the same workspace usable again."""
    T = 4
    projs, host = _block(1024, 2816, T, seed=71)
    prog = mmf.Program(projs, T)
    for p in projs:
        p["y"].fill_(float("nan"))
    prog.ws[:256].zero_()
    prog.run()
    torch.cuda.synchronize()
    assert mmf.mmf_get_device_status() == 8          # MMF_ERR_PLAN
    assert all(torch.isnan(p["y"].float()).all() for p in projs)
    mmf.mmf_program_init(projs, T, 1e-8, prog.ws)
    prog.run()
    torch.cuda.synchronize()
    assert mmf.mmf_get_device_status() == 0
    _check_against_oracle(projs, host)
