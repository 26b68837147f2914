"""X streamed from storage (fgmm_em_step_file / _reader, fgmm_em_partial_file): chunks
read into pinned buffers, copied to the device staging buffers and processed there must
give bit-identical results to the same step on a device copy of X (the device path is
itself checked against the oracle elsewhere); a failing reader ends the step with
FGMM_ERR_IO and leaves the parameters and the handle usable."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _handle(K, D, prec):
    import ivf_quantizer_b200 as q
    g = q.GMM(K, D)
    g.set_precision({"fp32": q.PREC_FP32, "fp16x3": q.PREC_FP16X3, "auto": q.PREC_AUTO}[prec])
    return g


def _run(g, w, mu, var, n_steps, N, one_step):
    wd, md, vd = g.new_params(w, mu, var)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    lz = torch.empty(N, dtype=torch.float32, device="cuda")
    lls = []
    for _ in range(n_steps):
        one_step(g, wd, md, vd, ll, lz)
        lls.append(float(ll.item()))
    torch.cuda.synchronize()
    assert g.status() == 0
    return wd, md, vd, lz, lls


def _same(a, b):
    for ta, tb in zip(a[:4], b[:4]):
        assert torch.equal(ta, tb)
    assert a[4] == b[4]


def _write(path, X, header=0):
    with open(path, "wb") as f:
        f.write(b"\x7f" * header)
        if X.dtype == torch.bfloat16:
            f.write(X.contiguous().view(torch.int16).numpy().tobytes())
        else:
            f.write(X.contiguous().numpy().tobytes())


@pytest.mark.parametrize("prec", ["fp16x3", "auto"])
def test_file_stream_equals_device_across_chunks(tmp_path, prec):
    import ivf_quantizer_b200 as q
    N = q.CHUNK_POINTS * 2 + 4321                       # three chunks, ragged tail
    X = synth.generate("c1", N, seed=7)
    w, mu, var = synth.init_params(X, 16, seed=7)
    path = tmp_path / "x.f32"
    _write(path, X, header=64)                          # rows start after a 64-byte header
    Xd = X.cuda()
    a = _run(_handle(16, 16, prec), w, mu, var, 2, N,
             lambda g, *p: g.step(Xd, *p[:3], loglik=p[3], logz=p[4]))
    b = _run(_handle(16, 16, prec), w, mu, var, 2, N,
             lambda g, *p: g.step_file(path, N, *p[:3], offset=64, loglik=p[3], logz=p[4]))
    _same(a, b)


def test_file_stream_auto_redo_bf16(tmp_path):
    """AUTO steps that move collapsing components to the side path (the device's path
    decision is read back before each optional pass, which reads the file again), bf16."""
    X = synth.generate("table1", 3000, seed=2).to(torch.bfloat16)
    w, mu, var = synth.init_params(X.float(), 256, seed=2)
    path = tmp_path / "x.bf16"
    _write(path, X)
    Xd = X.cuda()
    a = _run(_handle(256, 128, "auto"), w, mu, var, 3, 3000,
             lambda g, *p: g.step(Xd, *p[:3], loglik=p[3], logz=p[4]))
    b = _run(_handle(256, 128, "auto"), w, mu, var, 3, 3000,
             lambda g, *p: g.step_file(path, 3000, *p[:3], dtype=torch.bfloat16,
                                       loglik=p[3], logz=p[4]))
    _same(a, b)


def test_reader_and_partial_file(tmp_path):
    import ivf_quantizer_b200 as q
    N = q.CHUNK_POINTS + 999
    X = synth.generate("table1", N, seed=4)
    w, mu, var = synth.init_params(X, 64, seed=4)
    Xn = X.numpy()
    Xd = X.cuda()
    calls = []

    def read(row0, out):
        calls.append((row0, out.shape[0]))
        out[:] = Xn[row0:row0 + out.shape[0]]
        return True

    a = _run(_handle(64, 128, "fp16x3"), w, mu, var, 2, N,
             lambda g, *p: g.step(Xd, *p[:3], loglik=p[3], logz=p[4]))
    b = _run(_handle(64, 128, "fp16x3"), w, mu, var, 2, N,
             lambda g, *p: g.step_reader(read, N, *p[:3], loglik=p[3], logz=p[4]))
    _same(a, b)
    # one pass per step, chunks in increasing row order
    assert calls == [(0, q.CHUNK_POINTS), (q.CHUNK_POINTS, 999)] * 2
    # the sharded partial from a file equals the device partial
    path = tmp_path / "x.f32"
    _write(path, X)
    g = _handle(64, 128, "fp16x3")
    wd, md, vd = g.new_params(w, mu, var)
    s_dev = g.partial(Xd, wd, md, vd)
    s_file = g.partial_file(path, N, wd, md, vd)
    torch.cuda.synchronize()
    assert torch.equal(s_dev, s_file)


def test_failing_reader_and_missing_file(tmp_path):
    import ivf_quantizer_b200 as q
    from ivf_quantizer_b200._lib import FgmmError
    N = q.CHUNK_POINTS + 17
    X = synth.generate("c1", N, seed=3)
    w, mu, var = synth.init_params(X, 16, seed=3)
    g = _handle(16, 16, "auto")
    wd, md, vd = g.new_params(w, mu, var)
    before = (wd.clone(), md.clone(), vd.clone())

    def bad(row0, out):
        return row0 == 0          # the second chunk fails

    with pytest.raises(FgmmError) as ei:
        g.step_reader(bad, N, wd, md, vd)
    assert ei.value.code == q._lib.ERR_IO
    with pytest.raises(FgmmError) as ei:
        g.step_file(tmp_path / "missing.f32", N, wd, md, vd)
    assert ei.value.code == q._lib.ERR_IO
    short = tmp_path / "short.f32"
    _write(short, X[:1000])       # the file ends before the N rows do
    with pytest.raises(FgmmError) as ei:
        g.step_file(short, N, wd, md, vd)
    assert ei.value.code == q._lib.ERR_IO
    torch.cuda.synchronize()
    for t0, t1 in zip(before, (wd, md, vd)):
        assert torch.equal(t0, t1)            # parameters untouched
    # the handle still works
    g.step(X.cuda(), wd, md, vd)
    g.check_status()
    g.close()
