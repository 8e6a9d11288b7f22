"""The binding checks every tensor argument against the cache (or the MoBA layout)
before anything reaches the library: a tensor of the wrong shape, dtype or layout
raises KvcrArgError and nothing is launched.  These run without a GPU: shape and
dtype are checked before the device, and a CPU tensor of the right shape is refused
for not being a CUDA tensor."""
import pytest
import torch

from kv_cache_chunk_ring_b200 import kvcr


@pytest.fixture(scope="module", autouse=True)
def _built():
    from kv_cache_chunk_ring_b200 import build
    build.build()


T, H, D = 12, 3, 64


@pytest.fixture()
def cache():
    return kvcr.Cache(1, 2, T, H, D, 2, rope=None, bookkeeping_only=True)


def _t(*shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def _raises(fn, code, text):
    launches = kvcr.kvcr_launch_count()
    with pytest.raises(kvcr.KvcrArgError) as e:
        fn()
    assert e.value.code == code and text in str(e.value), str(e.value)
    assert kvcr.kvcr_launch_count() == launches


def test_chunk_attention_shapes(cache):
    n = 2 * T
    good = dict(q=_t(n, H, D), k=_t(n, H, D), v=_t(n, H, D), o=_t(n, H, D))

    def call(**kw):
        a = dict(good, **kw)
        return lambda: kvcr.chunk_attention_fwd(cache.handle, a["q"], a["k"], a["v"], [0, 1],
                                                a["o"], kw.get("lse"))
    _raises(call(k=_t(n - 1, H, D)), kvcr.KVCR_ESHAPE, "k_cur has shape")
    _raises(call(v=_t(n, H + 1, D)), kvcr.KVCR_ESHAPE, "v_cur has shape")
    _raises(call(o=_t(n - T, H, D)), kvcr.KVCR_ESHAPE, "o has shape")
    _raises(call(q=_t(n, H, 2 * D), o=_t(n, H, 2 * D)), kvcr.KVCR_ESHAPE, "q has shape")
    _raises(call(o=_t(n, H, D, dtype=torch.float32)), kvcr.KVCR_EINVAL, "o has dtype")
    _raises(call(lse=_t(n, H, dtype=torch.float32)), kvcr.KVCR_ESHAPE, "lse has shape")
    _raises(call(lse=_t(H, n, dtype=torch.bfloat16)), kvcr.KVCR_EINVAL, "lse has dtype")
    _raises(call(k=_t(n, D, H).transpose(1, 2)), kvcr.KVCR_EINVAL, "contiguous")
    _raises(call(), kvcr.KVCR_EINVAL, "must be a CUDA tensor")
    _raises(lambda: kvcr.chunk_attention_fwd_static_scratch(
        cache.handle, good["q"], good["k"], _t(1, H, D), [0, 1], good["o"]),
        kvcr.KVCR_ESHAPE, "v_cur has shape")
    _raises(lambda: cache.attention(_t(n, H, D), _t(n, H, D), _t(n, H, D), [0, 1],
                                    out=_t(n + 1, H, D)), kvcr.KVCR_ESHAPE, "o has shape")


def test_rope_cache_needs_one_query_per_chunk_token():
    c = kvcr.Cache(1, 2, T, H, D, 2, rope=kvcr.kvcr_rope(3, 4, 12, 10, 10, 10000.0),
                   bookkeeping_only=True)
    n = 2 * T
    _raises(lambda: kvcr.chunk_attention_fwd(c.handle, _t(n - 1, H, D), _t(n, H, D),
                                             _t(n, H, D), [0, 1], _t(n - 1, H, D)),
            kvcr.KVCR_ESHAPE, "with RoPE")


def test_append_and_aux_shapes(cache):
    _raises(lambda: cache.append(_t(T, H, D), _t(2 * T, H, D), [0, 1]), kvcr.KVCR_ESHAPE,
            "k has shape")
    _raises(lambda: cache.append(_t(2 * T, H, D), _t(2 * T, H, D, dtype=torch.float32), [0, 1]),
            kvcr.KVCR_EINVAL, "v has dtype")
    _raises(lambda: kvcr.kv_cache_set_aux(cache.handle, _t(T, H, D), _t(T, H, D - 1), None, 1),
            kvcr.KVCR_ESHAPE, "v has shape")
    other = kvcr.Cache(1, 2, T, H, D, 2, rope=None, bookkeeping_only=True)
    _raises(lambda: kvcr.append_batch([cache, other], [_t(T, H, D)] * 2,
                                      [_t(T, H, D), _t(T + 1, H, D)], [0]),
            kvcr.KVCR_ESHAPE, "[1] v has shape")


def test_destroyed_handle_refused():
    c = kvcr.Cache(1, 2, T, H, D, 2, rope=None, bookkeeping_only=True)
    h = c.handle
    kvcr.kv_cache_destroy(h)
    c.handle = None
    _raises(lambda: kvcr.chunk_attention_fwd(h, _t(T, H, D), _t(T, H, D), _t(T, H, D), [0],
                                             _t(T, H, D)), kvcr.KVCR_EINVAL, "unknown")


def test_moba_shapes():
    n, c, m = 2, 100, 1
    L = (2 * n + m) * c
    x = _t(L, 2, 128)
    _raises(lambda: kvcr.moba_attention_fwd(x, _t(L - 1, 2, 128), x, n, c, m, x),
            kvcr.KVCR_ESHAPE, "k has shape")
    _raises(lambda: kvcr.moba_attention_fwd(_t(L + 1, 2, 128), x, x, n, c, m, x),
            kvcr.KVCR_ESHAPE, "q has shape")
    _raises(lambda: kvcr.moba_attention_fwd(x, x, x, n, c, m, x, _t(L, 2, dtype=torch.float32)),
            kvcr.KVCR_ESHAPE, "lse has shape")
    lse = _t(2, L, dtype=torch.float32)
    _raises(lambda: kvcr.moba_attention_bwd(x, x, x, x, x, lse, n, c, m, x, _t(L, 2, 64), x),
            kvcr.KVCR_ESHAPE, "dk has shape")
    _raises(lambda: kvcr.moba_attention_bwd(x, x, x, x, x, None, n, c, m, x, x, x),
            kvcr.KVCR_EINVAL, "lse")
    _raises(lambda: kvcr.moba_attention_bwd(x, x, x, x, x, lse, n, c, m, x, x, x),
            kvcr.KVCR_EINVAL, "must be a CUDA tensor")
