"""One sequence split into chunks (sequence parallelism), on one GPU: every
chunk's carry (end state from zero, sum of Delta) is computed by the CUDA
library, the carries are stacked as an all-gather would deliver them, each
chunk's entering state is composed, and the chunks are scanned again from
there; the concatenated result equals the fp64 oracle's scan of the whole
sequence. The ranks run one after another here (this machine has one GPU);
the multi-process exchange itself is covered on CPU by test_dist_gloo.py."""
import numpy as np
import pytest
import torch

import ssm_inputs as gen
from tests.gpu_util import TOL, dev, host, oracle_scan, rel_err

pytestmark = pytest.mark.gpu


def _chunk(inp, a, b):
    return {k: (dev(np.ascontiguousarray(v[:, a:b])) if k in ("x", "delta", "z", "B", "C") and v is not None
                else dev(v)) for k, v in inp.items()}


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("cuts", [(0, 150, 300), (0, 64, 65, 200, 300), (0, 37, 111, 190, 256, 300)],
                         ids=["2", "4_with_one_step_chunk", "5_uneven"])
def test_split_sequence_matches_full_scan(io, cuts):
    from selective_state_space_39_b200.seqpar import chunk_carry, entering_state
    from selective_state_space_39_b200 import ssm_scan_fwd
    inp = gen.make_scan_inputs(2, 300, 200, 16, io, 31, with_h0=True)
    chunks = [_chunk(inp, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    carries = [chunk_carry(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                           delta_bias=c["delta_bias"]) for c in chunks]
    hend_all = torch.stack([e for e, _ in carries])
    dsum_all = torch.stack([s for _, s in carries])
    ys, h_last = [], None
    for r, c in enumerate(chunks):
        h_in = entering_state(r, c["A"], hend_all, dsum_all, h0=c["h0"])
        y, h_last = ssm_scan_fwd(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                                 delta_bias=c["delta_bias"], h0=h_in)
        ys.append(y)
    yr, hr = oracle_scan(inp, io)
    ey, eh = rel_err(host(torch.cat(ys, dim=1)), yr), rel_err(host(h_last), hr)
    print(f"{io} cuts={cuts}: rel err y {ey:.3e} h_last {eh:.3e}")
    assert ey <= TOL[io] and eh <= TOL[io]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("softplus", [True, False])
def test_delta_sum_matches_definition(io, softplus):
    """sum_t softplus(delta + bias) (fp64 from the same rounded inputs)."""
    from selective_state_space_39_b200 import ssm_delta_sum
    inp = gen.make_scan_inputs(3, 500, 130, 16, io, 33)
    got = host(ssm_delta_sum(dev(inp["delta"]), dev(inp["delta_bias"]), softplus=softplus))
    v = gen.as_float(inp["delta"], io).astype(np.float64) + inp["delta_bias"].astype(np.float64)
    dt = np.where(v > 20, v, np.log1p(np.exp(np.minimum(v, 20)))) if softplus else v
    want = dt.sum(axis=1)
    assert rel_err(got, want) <= (1e-5 if io == "f32" else 1e-4)


def test_compose_of_no_chunks_is_h0():
    from selective_state_space_39_b200 import ssm_compose_carries
    inp = gen.make_scan_inputs(2, 4, 64, 16, "f32", 35, with_h0=True)
    hend = torch.zeros((3, 2, 64, 16), dtype=torch.float32, device="cuda")
    dsum = torch.zeros((3, 2, 64), dtype=torch.float32, device="cuda")
    h0 = dev(inp["h0"])
    assert torch.equal(ssm_compose_carries(0, dev(inp["A"]), hend, dsum, h0=h0), h0)
    assert not ssm_compose_carries(0, dev(inp["A"]), hend, dsum).any()


def test_state_only_scan_writes_no_y():
    """return_y=False: the final state equals the full scan's, and no y."""
    from selective_state_space_39_b200 import ssm_scan_fwd
    inp = gen.make_scan_inputs(2, 100, 96, 16, "bf16", 37, with_h0=True)
    d = {k: dev(v) for k, v in inp.items()}
    y, h1 = ssm_scan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                         delta_bias=d["delta_bias"], h0=d["h0"])
    y2, h2 = ssm_scan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                          delta_bias=d["delta_bias"], h0=d["h0"], return_y=False)
    assert y2 is None and torch.equal(h1, h2)
