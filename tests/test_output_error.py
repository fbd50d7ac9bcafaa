"""The module-output-error diagnostic (summary page "WUSH-KV：数据自适应变换的
KV Cache 低比特量化", 关键实验, first bullet): relative attention-output error
of the quantised cache for the identity, a randomised Hadamard rotation and a
random invertible transform, through the oracle (CPU) and through the library
(GPU).  The pages' 0.208 / 0.309 / 0.325 need model weights and data and stay
context; these tests pin what holds on the synthetic data."""
import numpy as np
import pytest

from bit_kv_cache_post_b200 import inputs as I
from oracle import wushkv_oracle as O

W = I.WORKLOADS["qwen3-8b-layer-b16-ctx8192"]


def _data(B=1, n=1024):
    k = np.stack([I.keys(W, 0, b, n) for b in range(B)])
    v = np.stack([I.values(W, 0, b, n) for b in range(B)])
    q = np.stack([I.queries(W, 0, b) for b in range(B)])
    return I.round_to(k, "bf16"), I.round_to(v, "bf16"), I.round_to(q, "bf16")


def test_hadamard_is_orthogonal():
    T, TinvT = I.hadamard_transforms(W, 0)
    for h in range(T.shape[0]):
        assert np.allclose(T[h].astype(np.float64) @ T[h].T.astype(np.float64), np.eye(128), atol=1e-6)
        assert np.array_equal(T[h], TinvT[h])


def test_geometric_mean_definition():
    x = np.array([0.5, 2.0, 1.0, 4.0])
    assert abs(O.geometric_mean(x) - (0.5 * 2.0 * 1.0 * 4.0) ** 0.25) < 1e-12


def test_errors_vanish_without_quantisation_error():
    """A cache of only fp16 window tokens (no packed token) returns attention
    over the fp16-rounded keys: the error is that of fp16 rounding alone."""
    k, v, q = _data(n=200)
    T, TinvT = I.hadamard_transforms(W, 0)
    e = O.output_errors(k, v, q, T, TinvT, O.CacheConfig(1, 8, 32, 200, bits=2))
    assert e.max() < 2e-3


def test_rotation_spreads_outliers():
    """Keys with x20 outlier channels: the QuEST clip range follows the token
    RMS, so without a rotation the outlier channels saturate and more bits do
    not help; a Hadamard rotation spreads them and the error falls with bits,
    below the identity's at every width."""
    k, v, q = _data()
    E = {}
    for name, (T, Ti) in (("identity", I.identity_transforms(W)), ("hadamard", I.hadamard_transforms(W, 0))):
        for bits in (2, 3, 4):
            E[name, bits] = O.geometric_mean(O.output_errors(k, v, q, T, Ti, O.CacheConfig(1, 8, 32, 1024, bits=bits)))
    for bits in (2, 3, 4):
        assert E["hadamard", bits] < 0.8 * E["identity", bits]
    assert E["hadamard", 2] > E["hadamard", 3] > E["hadamard", 4]


@pytest.mark.gpu
@pytest.mark.parametrize("arm", ["identity", "hadamard", "random"])
def test_library_errors_match_oracle(arm):
    """The same diagnostic through the library (bf16 inputs, bulk append
    through T, query transform, decode): geometric means within 5 % of the
    oracle's (k' rounding-boundary flips are the only difference)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_kv_cache_post_b200 import wushkv as wk
    k, v, q = _data(B=2)
    T, Ti = {"identity": I.identity_transforms(W), "hadamard": I.hadamard_transforms(W, 0),
             "random": I.key_transforms(W, 0)}[arm]
    for quantizer in (O.QUEST_INT, O.AFFINE_PCTCLIP):
        for bits in (2, 4):
            ocfg = O.CacheConfig(2, 8, 32, 1024, bits=bits, quantizer=quantizer)
            want = O.geometric_mean(O.output_errors(k, v, q, T, Ti, ocfg))
            cache = wk.Cache(wk.make_config(2, 8, 32, 1024, bits=bits, quantizer=quantizer))
            dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
            cache.append(dev(k).bfloat16(), dev(v).bfloat16(), dev(T))
            out = cache.decode(wk.query_transform(dev(q).bfloat16(), dev(Ti))).cpu().numpy()
            ref = np.empty_like(out, dtype=np.float64)
            for b in range(2):
                for h in range(8):
                    ref[b, 4 * h:4 * h + 4] = O.attention_f64(q[b, 4 * h:4 * h + 4], k[b, :, h], v[b, :, h],
                                                              1.0 / np.sqrt(128.0))
            got = O.geometric_mean(np.linalg.norm(out - ref, axis=-1) / np.linalg.norm(ref, axis=-1))
            assert abs(got - want) <= 0.05 * want, (arm, quantizer, bits, got, want)
