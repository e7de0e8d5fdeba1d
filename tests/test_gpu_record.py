"""tlc_compress_recorded: the per-call record (M, scale, non-zero count,
stream length) written by the compress kernels, against the oracle's own
steps (error feedback and magnitude, quantization, the whole compression).
Needs a B200."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gradient_traffic_compression_b200 as g
    g.lib()
    return g


def _recorded(g, x, s, err):
    n = x.size
    xt = torch.from_numpy(x).cuda()
    et = torch.from_numpy(err.copy()).cuda()
    out = torch.empty(g.tlc_compress_bound(n), dtype=torch.uint8, device="cuda")
    ln = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rec = torch.full((24,), 0xEE, dtype=torch.uint8, device="cuda")
    g.tlc_compress_recorded(xt, s, et, out, ln, rec, st)
    torch.cuda.synchronize()
    L = int(ln.item())
    return int(st.item()), g.record_fields(rec), out[:L].cpu().numpy(), et.cpu().numpy()


def _oracle_record(x, s, err):
    xp = oracle.error_feedback(x, err)
    rc, M = oracle.magnitude(xp)
    rc_c, stream, err2 = oracle.compress(x, s, err)
    if rc:
        return rc, {"m_bits": None, "scale": 0.0, "length": 0}, None, None
    rc_q, q, _, scale = oracle.quantize(xp, M, s)
    assert rc_q == 0
    return rc_c, {"m_bits": int(np.float32(M).view(np.uint32)), "scale": float(scale),
                  "nonzeros": int(np.count_nonzero(q)), "length": int(stream.size)}, stream, err2


@pytest.mark.parametrize("case", ["config1", "config3_2^22", "deferred", "all_zero"])
def test_record_matches_the_oracle(g, case):
    if case == "config1":
        x, s = synth.flat_tensor(1), synth.CONFIGS[1]["s"]
        err = np.zeros(x.size, np.float32)
    elif case == "config3_2^22":
        x, s = synth.flat_tensor(3, n=1 << 22), 1.9
        err = synth.laplace(synth.key_for(901, 1), x.size, 2e-5)
    elif case == "deferred":          # 384 compress tiles or more: placement kernel
        n = 384 * 20480 + 999
        x = synth.normal(synth.key_for(902, 0), n, 1e-3)
        x[synth.bernoulli(synth.key_for(902, 1), n, 0.6)] = 0.0
        s, err = 1.5, np.zeros(n, np.float32)
    else:
        x, s, err = np.zeros(1000, np.float32), 1.2, np.zeros(1000, np.float32)
    rc, rec, stream, e2 = _recorded(g, x, s, err)
    rc_o, want, stream_o, e_o = _oracle_record(x, s, err)
    assert rc == rc_o == 0
    assert rec == want, (rec, want)
    assert np.array_equal(stream, stream_o)
    assert np.array_equal(e2.view(np.uint32), e_o.view(np.uint32))


def test_record_of_a_nonfinite_step(g):
    x = synth.normal(synth.key_for(903, 0), 50_000, 1e-3)
    x[777] = np.inf
    rc, rec, stream, e2 = _recorded(g, x, 1.5, np.zeros(x.size, np.float32))
    assert rc == 2
    assert rec["m_bits"] >= 0x7F800000 and rec["scale"] == 0.0 and rec["length"] == 0
    assert stream.size == 0
