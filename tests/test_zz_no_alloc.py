"""svdq_quantize_act_noalloc against svdq_quantize_act on the GPU.

The allocation-free entry point is for callers that cannot hand the library
working memory: a serving runtime or a plugin whose allocator sized all device
memory before the first request, where an allocation mid-step would escape that
budget, could block or synchronise the device, and could fail under memory
pressure. It keeps the K splits' partial down-projections in a static device
array instead of the caller's workspace; on the same inputs
it must return the same bytes as the regular call, on two calls in a row, each
right after a call on another activation of the same shape (so every compared
call finds the array holding someone else's partial sums). This file is
collected last so it also runs after every other GPU test in one session.
"""

import numpy as np
import pytest

import workloads as WL
from oracle import formats as F
from oracle import layout as LO
from tests import svdq_cases as C

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_quantized_diffusion_b200 as bq
    return bq


CASES = [
    # K split into several ranges (svdq_xl1_splits > 1), ragged rows
    WL.custom_svdq("split_ragged", 300, 1024, 272, 32, seed=41),
    # the QKV activation shape: 4 splits of 768 columns
    WL.custom_svdq("qkv_rows", 4608, 3072, 64, 32, seed=42),
    WL.custom_svdq("int4_split", 520, 2048, 128, 48, fmt="int4", seed=43),
    WL.custom_svdq("rank0", 130, 512, 64, 0, seed=44),
]


@pytest.mark.parametrize("shape", CASES, ids=lambda s: s.name)
def test_noalloc_matches_the_regular_call_twice(bq, shape):
    d = WL.svdq_inputs(shape)
    M, K, r = shape.M, shape.K, shape.r
    rng = np.random.default_rng(shape.seed)
    X = C.bf16_tensor(d["X"])
    si = C.f32_tensor(F.rn32(rng.uniform(0.2, 2.0, K)))
    L1s = None
    if r:
        L1 = F.bf16_round(rng.normal(0, 0.05, (K, r)))
        L1s = C.bf16_tensor(F.bf16_bits(LO.lowrank_operand(L1, F.rn32(si.cpu().numpy().astype(np.float64)))))
    want = bq.svdq_quantize_act(X, L1s, si, fmt=shape.fmt)
    # another activation of the same shape: the call before each compared call
    # leaves its own partial sums in the static array, so a compared call that
    # skipped writing part of the array would read them and differ
    X_other = C.bf16_tensor(WL.to_bf16_bits(rng.standard_normal((M, K)) * 3.0))
    assert bq.svdq_check_device_status() == 0
    for call in range(2):
        bq.svdq_quantize_act_noalloc(X_other, L1s, si, fmt=shape.fmt)
        got = bq.svdq_quantize_act_noalloc(X, L1s, si, fmt=shape.fmt)
        assert bq.svdq_check_device_status() == 0
        for name, a, b in zip(("codes", "scales", "xl1"), got, want):
            if b is None:
                assert a is None
                continue
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), f"call {call}: {name} differs"


def test_noalloc_rejects_a_request_beyond_its_array(bq):
    # (S - 1) * M * r floats must fit in 2^21: M = 4608, K = 3072 gives S = 4,
    # so r = 256 needs 3 * 4608 * 256 = 3.5 M floats
    M, K, r = 4608, 3072, 256
    assert bq.svdq_xl1_splits(M, K, r) == 4
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    L1s = torch.zeros((2, r, K), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bq.SvdqError) as e:
        bq.svdq_quantize_act_noalloc(X, L1s, None)
    assert e.value.status == 3  # SVDQ_ERR_UNSUPPORTED
    assert bq.svdq_check_device_status() == 0
