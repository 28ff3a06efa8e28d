"""moe_permute_noalloc against moe_permute, through the C ABI.

moe_permute_noalloc serves callers that cannot allocate device memory (a plug-in
inside a framework that owns all device memory, or code with a fixed footprint):
it keeps its histogram scratch in a 2 MiB array inside the library instead of a
caller workspace.  Its outputs must equal moe_permute's exactly (integers), on
consecutive calls that reuse the built-in scratch.  This file is collected last
so that a failure here does not hide the other tests.
"""
import numpy as np
import pytest
import torch

import mixture_experts_lora_b200 as ml

from gpu_common import ensure_built

pytestmark = pytest.mark.gpu


def _outputs(T, k, E):
    return (torch.empty(E, dtype=torch.int32, device="cuda"),
            torch.empty(E + 1, dtype=torch.int32, device="cuda"),
            torch.full((T * k,), -1, dtype=torch.int32, device="cuda"),
            torch.full((T * k,), -1, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("T,k,E", [(4096, 8, 128), (1500, 3, 7)])
def test_permute_noalloc_matches_permute_on_consecutive_calls(T, k, E):
    ensure_built()
    ws = torch.empty(ml.moe_workspace_bytes(ml.make_dims(T, 64, 64, E, k, 16, 1.0)),
                     dtype=torch.uint8, device="cuda")
    for call in range(2):
        rng = np.random.default_rng(100 * call + E)
        ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        if call == 1:
            ids[: T // 2, 0] = E - 1          # a hot expert on the second call
            ids[: T // 2, 1:][ids[: T // 2, 1:] == E - 1] = 0
        ids_d = torch.from_numpy(ids).cuda()
        ref = _outputs(T, k, E)
        got = _outputs(T, k, E)
        ml.moe_permute(ids_d, E, *ref, ws)
        ml.moe_permute_noalloc(ids_d, E, *got)
        torch.cuda.synchronize()
        assert ml.moe_get_device_error() == ml.MOE_OK
        for a, b in zip(ref, got):
            assert torch.equal(a, b), f"call {call}"


def test_permute_noalloc_rejects_oversized_problem():
    ensure_built()
    E, k = 1024, 8
    scratch_ints, chunk = 1 << 19, 512       # built-in scratch, pairs per histogram chunk
    T = (scratch_ints // E + 1) * chunk // k  # one chunk more than the scratch holds
    ids = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    outs = _outputs(T, k, E)
    with pytest.raises(ml.MoEError) as e:
        ml.moe_permute_noalloc(ids, E, *outs)
    assert e.value.status == ml.MOE_ERR_WORKSPACE


def test_permute_noalloc_at_the_exact_scratch_limit():
    # ceil(T*k / 512) * E == 2^19 histogram entries: the largest problem the built-in
    # scratch holds must be accepted and give moe_permute's outputs
    ensure_built()
    E, k, T = 1024, 8, 32768
    assert (T * k + 511) // 512 * E == 1 << 19
    rng = np.random.default_rng(7)
    ids = np.argsort(rng.random((T, E), dtype=np.float32), axis=1)[:, :k].astype(np.int32)
    ids_d = torch.from_numpy(ids).cuda()
    ws = torch.empty(ml.moe_workspace_bytes(ml.make_dims(T, 64, 64, E, k, 16, 1.0)),
                     dtype=torch.uint8, device="cuda")
    ref = _outputs(T, k, E)
    got = _outputs(T, k, E)
    ml.moe_permute(ids_d, E, *ref, ws)
    ml.moe_permute_noalloc(ids_d, E, *got)
    torch.cuda.synchronize()
    assert ml.moe_get_device_error() == ml.MOE_OK
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
