"""Host-side argument checks of the PyTorch calls, without a GPU.

Every tensor the kernels read or write through a raw pointer is checked for
dtype, exact shape, device and contiguity before anything is enqueued: a
too-small output or one on another GPU must be rejected on the host, never
reach a kernel.  Here the library is replaced by a recorder (no call reaches
libsbl.so) and tensors are CPU tensors that report themselves as CUDA ones,
so only the checks run."""
import pytest
import torch

from sparse_linear_layers_b200 import api


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append(name)
            return 0
        return call


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(api, "lib", r)
    monkeypatch.setattr(api, "_stream", lambda s: 0)
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: self.device.type == "cpu"))
    return r


T, K, O = 5, 64, 32


def _w():
    return api.PreparedWeights(torch.zeros((O, K // 4), dtype=torch.uint8), torch.ones(O), 2, 4, K)


def _x():
    return torch.zeros((T, K), dtype=torch.bfloat16)


def _ws():
    return torch.zeros(4096, dtype=torch.uint8)


def test_linear_accepts_matching_tensors(rec):
    api.sbl_linear(_x(), _w(), y=torch.empty((T, O)), acc_out=torch.empty((T, O), dtype=torch.int32),
                   workspace=_ws())
    assert rec.calls == ["sbl_linear_path"]


@pytest.mark.parametrize("kw", [
    dict(y=torch.empty((T, O - 1))),
    dict(y=torch.empty((T + 1, O))),
    dict(y=torch.empty((T, O), device="meta")),
    dict(y=torch.empty((O, T)).t()),
    dict(acc_out=torch.empty((T, O - 1), dtype=torch.int32)),
    dict(acc_out=torch.empty((T, O), dtype=torch.int64)),
    dict(acc_out=torch.empty((T, O), dtype=torch.int32, device="meta")),
    dict(workspace=torch.zeros((2, 64), dtype=torch.uint8)),
    dict(workspace=torch.zeros(64, dtype=torch.uint8, device="meta")),
])
def test_linear_rejects_bad_outputs(rec, kw):
    args = dict(y=torch.empty((T, O)), workspace=_ws())
    args.update(kw)
    with pytest.raises(ValueError):
        api.sbl_linear(_x(), _w(), **args)
    with pytest.raises(ValueError):
        api.sbl_linear_rmsnorm(_x(), _w(), torch.ones(K), **args)
    assert rec.calls == []


def test_linear_rejects_bad_weights(rec):
    w = _w()
    bad = [api.PreparedWeights(w.packed, torch.ones(O - 1), 2, 4, K),
           api.PreparedWeights(w.packed[:, :-1].contiguous(), w.row_scale, 2, 4, K),
           api.PreparedWeights(w.packed.to("meta"), w.row_scale, 2, 4, K)]
    for wb in bad:
        with pytest.raises(ValueError):
            api.sbl_linear(_x(), wb, y=torch.empty((T, O)), workspace=_ws())
    with pytest.raises(ValueError):
        api.sbl_linear(torch.zeros((T, K + 16), dtype=torch.bfloat16), w, workspace=_ws())
    with pytest.raises(ValueError):
        api.sbl_linear(torch.zeros((1, T, K), dtype=torch.bfloat16), w, workspace=_ws())
    with pytest.raises(ValueError):
        api.sbl_linear_rmsnorm(_x(), w, torch.ones(K - 16), y=torch.empty((T, O)), workspace=_ws())
    assert rec.calls == []


def test_backward_checks(rec):
    w, dY = _w(), torch.zeros((T, O))
    xq, s = torch.zeros((T, K), dtype=torch.int8), torch.ones(T)
    api.sbl_linear_backward(dY, xq, s, w, dX=torch.empty((T, K)), dW=torch.empty((O, K)), tensor_cores=False)
    assert rec.calls == ["sbl_linear_backward"]
    rec.calls.clear()
    api.sbl_linear_backward(dY, xq, s, w, dX=torch.empty((T, K)), dW=torch.empty((O, K)),
                            workspace=torch.empty(64, dtype=torch.uint8))
    assert rec.calls == ["sbl_linear_backward_ws"]
    rec.calls.clear()
    for kw in (dict(dW=torch.empty((O - 1, K))), dict(dW=torch.empty((O, K - 16))), dict(dX=torch.empty((T, K - 1))),
               dict(dX=torch.empty((T, K), device="meta")), dict(dW=torch.empty((O, K), dtype=torch.float64))):
        args = dict(dX=torch.empty((T, K)), dW=torch.empty((O, K)))
        args.update(kw)
        with pytest.raises(ValueError):
            api.sbl_linear_backward(dY, xq, s, w, **args)
    with pytest.raises(ValueError):
        api.sbl_linear_backward(dY, xq.to("meta"), s, w)
    with pytest.raises(ValueError):
        api.sbl_linear_backward(dY, xq, s, w, workspace=torch.empty(64, dtype=torch.uint8, device="meta"))
    assert rec.calls == []


def test_prepare_and_quant_checks(rec):
    W = torch.zeros((O, K))
    out = api.PreparedWeights(torch.empty((O, K // 4), dtype=torch.uint8), torch.empty(O), 2, 4, K,
                              torch.empty((O, K // 8), dtype=torch.uint8))
    api.sbl_prepare_weights(W, 2, 4, out=out)
    assert rec.calls == ["sbl_prepare_weights_ex"]
    rec.calls.clear()
    bad = [api.PreparedWeights(torch.empty((O, K // 4 - 1), dtype=torch.uint8), torch.empty(O), 2, 4, K),
           api.PreparedWeights(torch.empty((O, K // 4), dtype=torch.uint8), torch.empty(O), 2, 4, K,
                               torch.empty((O, K // 16), dtype=torch.uint8)),
           api.PreparedWeights(torch.empty((O - 1, K // 4), dtype=torch.uint8), torch.empty(O - 1), 2, 4, K)]
    for o in bad:
        with pytest.raises(ValueError):
            api.sbl_prepare_weights(W, 2, 4, out=o)
    with pytest.raises(ValueError):
        api.sbl_rmsnorm_quant_act(_x(), torch.ones(K, device="meta"))
    with pytest.raises(ValueError):
        api.sbl_quant_act(torch.zeros(K, dtype=torch.bfloat16))
    assert rec.calls == []


def test_linear_q_checks(rec):
    w = _w()
    xq, s = torch.zeros((T, K), dtype=torch.int8), torch.ones(T)
    api.sbl_linear_q(xq, s, w, y=torch.empty((T, O)), acc_out=torch.empty((T, O), dtype=torch.int32),
                     workspace=_ws())
    assert rec.calls == ["sbl_linear_q"]
    rec.calls.clear()
    bad_inputs = [(xq.to(torch.uint8), s), (xq, torch.ones(T + 1)), (xq, s.double()), (xq, s.to("meta")),
                  (xq.to("meta"), s), (torch.zeros((T, K + 64), dtype=torch.int8), s),
                  (torch.zeros((K, T), dtype=torch.int8).t(), s)]
    for a, b in bad_inputs:
        with pytest.raises(ValueError):
            api.sbl_linear_q(a, b, w, y=torch.empty((T, O)), workspace=_ws())
    for kw in (dict(y=torch.empty((T, O + 1))), dict(acc_out=torch.empty((T, O), dtype=torch.int64)),
               dict(workspace=torch.zeros(64, dtype=torch.uint8, device="meta"))):
        args = dict(y=torch.empty((T, O)), workspace=_ws())
        args.update(kw)
        with pytest.raises(ValueError):
            api.sbl_linear_q(xq, s, w, **args)
    assert rec.calls == []


@pytest.mark.parametrize("k,contraction,other", [(64, "sbl_linear_q", "sbl_linear_path"),
                                                   (48, "sbl_linear_path", "sbl_linear_q")])
def test_training_forward_quantises_once(rec, k, contraction, other):
    """The training layer's forward contracts the x_q it keeps for the backward
    (sbl_linear_q) when K % 64 == 0, else lets sbl_linear quantise x."""
    from sparse_linear_layers_b200 import train
    x = torch.zeros((T, k), dtype=torch.bfloat16)
    train.SparseBitLinearFunction.apply(x, torch.zeros((O, k)), 2, 4, False, True)
    assert rec.calls.count("sbl_quant_act") == 1
    assert contraction in rec.calls and other not in rec.calls
    assert rec.calls[-1] == "sbl_device_status"
