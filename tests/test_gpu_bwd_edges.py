"""GPU parity of the backward pass on the method's degenerate inputs, every
gradient against the fp64 oracle's adjoint loop (bounds as in the other
backward tests: 1e-4 fp32 io, 2e-2 bf16 io, relative to max|ref|):

  * x = 0 on a run of steps that crosses segment boundaries (padding tokens);
  * Delta = 0 with softplus off: the state is kept (the gradients of the
    decays and of Delta still flow);
  * delta + bias = 60: memoryless steps, every decay underflows;
  * A = 0: the state is h0 plus a running sum;
  * |h0| ~ 1e4 with an upstream dh_last;

with the default plan and with three segments (the checkpoints, the carry
composition and the segment-entering adjoints all take part)."""
import numpy as np
import pytest

import ssm_inputs as gen
from tests.test_gpu_bwd import check_all, gpu_bwd, oracle_bwd

pytestmark = pytest.mark.gpu

BATCH, L, DIM, N = 2, 120, 128, 16
IOS = ["f32", "bf16"]
SEGS = [None, "3"]


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    monkeypatch.delenv("SSM_SCAN_BWD_SEGMENTS", raising=False)
    yield


def _case(io, seed):
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, seed, with_h0=True)
    grads = gen.make_grad_inputs(BATCH, L, DIM, N, io, seed)
    return inp, grads


def _to_io(a, io):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return gen.f32_to_bf16_bits(a) if io == "bf16" else a


def _as_f32(a, io):
    return gen.bf16_bits_to_f32(a) if io == "bf16" else np.asarray(a, dtype=np.float32)


def _run(monkeypatch, inp, grads, io, segments, what, softplus=True):
    if segments:
        monkeypatch.setenv("SSM_SCAN_BWD_SEGMENTS", segments)
    g = gpu_bwd(inp, grads, softplus=softplus)
    check_all(g, oracle_bwd(inp, grads, io, softplus=softplus), io, f"{what} {io} seg={segments}")


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_bwd_zero_x_run(monkeypatch, io, segments):
    inp, grads = _case(io, 801)
    x = _as_f32(inp["x"], io).copy()
    x[:, 30:75, :] = 0.0
    inp["x"] = _to_io(x, io)
    _run(monkeypatch, inp, grads, io, segments, "x = 0 on steps 30-74")


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_bwd_delta_zero_keeps_state(monkeypatch, io, segments):
    inp, grads = _case(io, 802)
    inp["delta"] = _to_io(np.zeros((BATCH, L, DIM)), io)
    inp["delta_bias"] = None
    _run(monkeypatch, inp, grads, io, segments, "Delta = 0", softplus=False)


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_bwd_huge_delta_on_some_steps(monkeypatch, io, segments):
    inp, grads = _case(io, 803)
    d = _as_f32(inp["delta"], io).copy()
    d[:, ::5, :] = 60.0
    d[:, 50:70, :] = 60.0
    inp["delta"] = _to_io(d, io)
    _run(monkeypatch, inp, grads, io, segments, "Delta = 60 on some steps")


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_bwd_A_zero(monkeypatch, io, segments):
    inp, grads = _case(io, 804)
    inp["A"] = np.zeros((DIM, N), np.float32)
    _run(monkeypatch, inp, grads, io, segments, "A = 0")


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_bwd_large_h0(monkeypatch, io, segments):
    inp, grads = _case(io, 805)
    inp["h0"] = (inp["h0"] * 1e4).astype(np.float32)
    _run(monkeypatch, inp, grads, io, segments, "|h0| ~ 1e4")
