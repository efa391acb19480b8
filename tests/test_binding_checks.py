"""The Python binding's own argument checks, which run before any C call (CPU only):
tensors must be CUDA tensors of the documented dtype and rank."""
import pytest
import torch

import invariant_deterministic_04_b200 as bi


def test_cpu_tensors_are_refused_before_the_library_is_called():
    x = torch.zeros((4, 512), dtype=torch.bfloat16)
    w = torch.zeros(512, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="CUDA"):
        bi.rmsnorm(x, w)
    with pytest.raises(TypeError, match="CUDA"):
        bi.matmul(x, torch.zeros((64, 512), dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="CUDA"):
        bi.log_softmax(x)
    with pytest.raises(TypeError, match="CUDA"):
        bi.sample(x, torch.zeros(4, dtype=torch.int64), torch.zeros(4, dtype=torch.int64), 0.8)


def test_wrong_dtype_is_refused():
    class FakeCuda(torch.Tensor):  # a CPU tensor that claims to be on CUDA, to reach the dtype check
        @property
        def is_cuda(self):
            return True

    x = torch.zeros((4, 512), dtype=torch.float32).as_subclass(FakeCuda)
    with pytest.raises(TypeError, match="bfloat16"):
        bi.log_softmax(x)
    y = torch.zeros((4, 512, 3), dtype=torch.bfloat16).as_subclass(FakeCuda)
    with pytest.raises(ValueError, match="2 dims"):
        bi.row_mean(y)


# ---------------------------------------------------------------------------
# Every wrapper, run against a stand-in library on CPU tensors that claim to be on
# CUDA: the argument patterns the GPU tests, the benchmark and the decoder harness
# use are accepted and reach the right C entry point; caller outputs of the wrong
# shape or dtype, short index tensors and mixed devices are refused before any C
# call; a caller's stream becomes the current stream for the call.

import contextlib  # noqa: E402


class _FakeCuda(torch.Tensor):
    @property
    def is_cuda(self):
        return True


def _c(t):
    return t.as_subclass(_FakeCuda)


class _FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return 4096 if name.endswith("workspace_size") else 0
        return fn


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()
    entered = []

    class _S:
        cuda_stream = 0

    @contextlib.contextmanager
    def _dev(d):
        yield

    @contextlib.contextmanager
    def _stream(s):
        entered.append(s)
        yield

    monkeypatch.setattr(bi, "lib", lambda: lib)
    monkeypatch.setattr(torch.cuda, "device", _dev)
    monkeypatch.setattr(torch.cuda, "stream", _stream)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a: _S())
    lib.entered = entered
    return lib


def _bf(*shape):
    return _c(torch.zeros(shape, dtype=torch.bfloat16))


def _i32(*shape):
    return _c(torch.zeros(shape, dtype=torch.int32))


def test_every_wrapper_accepts_the_call_patterns_in_use(fake):
    x, w = _bf(6, 512), _bf(512)
    bi.rmsnorm(x, w)
    bi.rmsnorm(x, w, 1e-6, out=x)                                   # in place
    bi.rmsnorm(_bf(6, 1024)[:, :512], w, 1e-6, out=_bf(6, 1024)[:, 256:768])  # strided rows in and out
    a, W = _bf(5, 128), _bf(512, 128)
    bi.matmul(a, W)
    bi.matmul(a, W, out=_bf(8, 1024)[:5, 256:768])                  # strided output
    outs = bi.matmul_multi(a, [W, _bf(256, 128), _bf(64, 128)])
    assert [tuple(c.shape) for c in outs] == [(5, 512), (5, 256), (5, 64)]
    wide = _bf(5, 768)
    bi.matmul_multi(a, [W, _bf(256, 128)], outs=[wide[:, :512], wide[:, 512:]])  # column ranges of one output
    q, kc = _bf(3, 32, 128), _bf(10, 8, 16, 128)
    pt, lens = _i32(3, 4), _i32(3)
    bi.attention_decode(q, kc, kc, pt, lens)
    bi.attention_decode(q, kc, kc, pt, lens, out=_bf(3, 32, 128), workspace=_c(torch.zeros(4096, dtype=torch.uint8)))
    bi.attention_decode_static(q, kc, kc, pt, lens)
    fused = _bf(7, 48 * 128)
    qv = fused[:, : 32 * 128].view(7, 32, 128)                        # q part of a fused QKV row
    kv_new = fused[:, 32 * 128: 40 * 128].view(7, 8, 128)
    qs, qp = _i32(3, 7)[0], _i32(3, 7)[1]
    bi.attention_prefill(qv, qs, qp, kc, kc, pt)
    bi.attention_prefill(_bf(7, 32, 128), qs, qp, kc, kc, pt, out=_bf(7, 32, 128),
                         workspace=_c(torch.zeros(4096, dtype=torch.uint8)))
    bi.attention_prefill_tc(_bf(7, 32, 128), 0, 0, kc, kc, pt)
    bi.attention_prefill_tc(_bf(7, 32, 128), 0, 5, kc, kc, pt, out=_bf(7, 32, 128))
    bi.kv_append(kv_new, kv_new, qs, qp, kc, kc, pt)
    bi.rope(qv, qp, _c(torch.zeros((384, 64, 2), dtype=torch.float32)))
    bi.gather_rows(_bf(100, 256), _i32(9))
    bi.swiglu(_bf(4, 2 * 256))
    h = _bf(9, 256)
    bi.add(h, _bf(9, 256), out=h)
    bi.add(h, _bf(9, 256))
    hh, Wl = _bf(4, 128), _bf(512, 128)
    bi.lmhead_argmax(hh, Wl, 0.5, want_logits=True)
    bi.lmhead_argmax(hh, Wl, 0.5, tokens=_i32(4), recomputed=_i32(4), workspace=_c(torch.zeros(64, dtype=torch.uint8)))
    lg = _bf(64, 1000)
    y = _c(torch.zeros((64, 1000), dtype=torch.float32))
    bi.log_softmax(lg)
    bi.log_softmax(lg[:8], out=y[:8])
    bi.token_logprob(lg, _i32(64), out=_c(torch.zeros(64, dtype=torch.float32)))
    bi.row_mean(lg, out=_c(torch.zeros(64, dtype=torch.float32)))
    seeds, steps = _c(torch.zeros(64, dtype=torch.int64)), _c(torch.zeros(64, dtype=torch.int64))
    bi.sampling_uniforms(seeds, steps, 1000)
    bi.sample(lg, seeds, steps, 0.8, out=_i32(64))
    names = set(fake.calls)
    for n in ("bi_rmsnorm", "bi_matmul", "bi_matmul_multi", "bi_attention_decode", "bi_attention_decode_static", "bi_attention_prefill",
              "bi_attention_prefill_tc", "bi_kv_append", "bi_rope", "bi_gather_rows", "bi_swiglu", "bi_add",
              "bi_lmhead_argmax", "bi_log_softmax", "bi_token_logprob", "bi_row_mean", "bi_sampling_uniforms",
              "bi_sample"):
        assert n in names, n
    assert fake.entered == []  # no stream given: the current stream is used as it is


def test_wrong_outputs_and_index_tensors_are_refused_before_the_c_call(fake):
    x, w = _bf(6, 512), _bf(512)
    cases = [
        (ValueError, lambda: bi.rmsnorm(x, w, out=_bf(5, 512))),
        (ValueError, lambda: bi.matmul(_bf(5, 128), _bf(512, 128), out=_bf(5, 256))),
        (TypeError, lambda: bi.matmul(_bf(5, 128), _bf(512, 128), out=_c(torch.zeros((5, 512))))),
        (ValueError, lambda: bi.matmul(_bf(5, 128), _bf(512, 128), out=_bf(512, 5).t())),  # columns strided
        (ValueError, lambda: bi.matmul_multi(_bf(5, 128), [])),                            # no product
        (ValueError, lambda: bi.matmul_multi(_bf(5, 128), [_bf(64, 128)] * 4)),            # more than three
        (ValueError, lambda: bi.matmul_multi(_bf(5, 128), [_bf(64, 128), _bf(64, 256)])),  # inner dims differ
        (ValueError, lambda: bi.matmul_multi(_bf(5, 128), [_bf(64, 128)], outs=[])),       # outs count
        (ValueError, lambda: bi.matmul_multi(_bf(5, 128), [_bf(64, 128)], outs=[_bf(5, 32)])),  # out shape
        (ValueError, lambda: bi.matmul_multi(_bf(5, 128), [_bf(128, 64).t()])),             # W rows strided
        (ValueError, lambda: bi.attention_decode(_bf(3, 32, 128), _bf(10, 8, 16, 128), _bf(10, 8, 16, 128),
                                                 _i32(3, 4), _i32(3), out=_bf(2, 32, 128))),
        (ValueError, lambda: bi.attention_prefill_tc(_bf(7, 32, 128), 0, 0, _bf(10, 8, 16, 128), _bf(10, 8, 16, 128),
                                                     _i32(1, 4), out=_bf(7, 32, 128)[:, :, :64])),
        (ValueError, lambda: bi.kv_append(_bf(7, 8, 128), _bf(7, 8, 128), _i32(6), _i32(7), _bf(10, 8, 16, 128),
                                          _bf(10, 8, 16, 128), _i32(1, 4))),
        (ValueError, lambda: bi.kv_append(_bf(7, 8, 128), _bf(7, 8, 128), _i32(7), _i32(7), _bf(10, 8, 16, 64),
                                          _bf(10, 8, 16, 64), _i32(1, 4))),
        (ValueError, lambda: bi.rope(_bf(7, 32, 128), _i32(6), _c(torch.zeros((384, 64, 2))))),
        (ValueError, lambda: bi.gather_rows(_bf(100, 256), _i32(9), out=_bf(9, 128))),
        (ValueError, lambda: bi.swiglu(_bf(4, 512), out=_bf(4, 512))),
        (ValueError, lambda: bi.add(_bf(9, 256), _bf(9, 256), out=_bf(9, 128))),
        (ValueError, lambda: bi.lmhead_argmax(_bf(4, 128), _bf(512, 128), tokens=_i32(3))),
        (TypeError, lambda: bi.lmhead_argmax(_bf(4, 128), _bf(512, 128), recomputed=_bf(4))),
        (ValueError, lambda: bi.lmhead_argmax(_bf(4, 128), _bf(512, 128), logits_fp32=_c(torch.zeros((4, 511))))),
        (ValueError, lambda: bi.lmhead_argmax(_bf(4, 128), _bf(512, 64))),
        (TypeError, lambda: bi.lmhead_argmax(_bf(4, 128), _bf(512, 128), workspace=torch.zeros(64, dtype=torch.uint8))),
        (ValueError, lambda: bi.log_softmax(_bf(64, 1000), out=_c(torch.zeros((64, 999))))),
        (ValueError, lambda: bi.token_logprob(_bf(64, 1000), _i32(63))),
        (ValueError, lambda: bi.row_mean(_bf(64, 1000), out=_c(torch.zeros(65)))),
        (ValueError, lambda: bi.sample(_bf(64, 1000), _c(torch.zeros(64, dtype=torch.int64)),
                                       _c(torch.zeros(64, dtype=torch.int64)), 0.8, out=_i32(65))),
        (ValueError, lambda: bi.sampling_uniforms(_c(torch.zeros(4, dtype=torch.int64)),
                                                  _c(torch.zeros(4, dtype=torch.int64)), 64, out=_c(torch.zeros((4, 63))))),
    ]
    for i, (err, call) in enumerate(cases):
        with pytest.raises(err):
            call()
        assert fake.calls == [], i


def test_tensors_on_two_devices_are_refused(fake):
    other = torch.zeros((512, 128), dtype=torch.bfloat16, device="meta").as_subclass(_FakeCuda)
    with pytest.raises(ValueError, match="all tensors must be on"):
        bi.matmul(_bf(5, 128), other)
    with pytest.raises(ValueError, match="all tensors must be on"):
        bi.rmsnorm(_bf(6, 512), _bf(512), out=torch.zeros((6, 512), dtype=torch.bfloat16,
                                                          device="meta").as_subclass(_FakeCuda))
    assert fake.calls == []


def test_a_stream_of_another_device_is_refused(fake):
    class _OtherStream:
        device = torch.device("meta")

    with pytest.raises(ValueError, match="stream is on"):
        bi.matmul(_bf(5, 128), _bf(512, 128), stream=_OtherStream())
    assert fake.calls == []


def test_a_callers_stream_is_current_for_the_call(fake):
    s = object()
    bi.matmul(_bf(5, 128), _bf(512, 128), stream=s)
    bi.attention_decode(_bf(3, 32, 128), _bf(10, 8, 16, 128), _bf(10, 8, 16, 128), _i32(3, 4), _i32(3), stream=s)
    bi.lmhead_argmax(_bf(4, 128), _bf(512, 128), stream=s)
    assert fake.entered == [s, s, s]
