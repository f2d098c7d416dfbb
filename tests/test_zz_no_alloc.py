"""GPU check of fp8_moe_route_noalloc, the routing entry point whose sort scratch is a
fixed device array inside the library instead of a caller workspace.  On two calls in a
row (different scores each time) it must give exactly what fp8_moe_route gives.  This
file is collected last, so in a full run it also exercises the array after every other
test has used the library in the same process; it passes on its own as well."""
import pytest
import torch

import fp8_block_scaled_12_b200 as F

pytestmark = pytest.mark.gpu

NAMES = ("ids", "w", "offsets", "row_token", "row_weight", "token_row")


@pytest.mark.parametrize("T,E,k", [(4096, 256, 8), (300, 64, 8), (64, 256, 8), (200, 1024, 4)])
def test_noalloc_route_matches_workspace_route(cuda_device, T, E, k):
    g = torch.Generator(device=cuda_device).manual_seed(T + E + k)
    for call in range(2):
        scores = torch.rand((T, E), generator=g, device=cuda_device)
        ref = F.moe_route(scores, k)
        got = F.moe_route_noalloc(scores, k)
        torch.cuda.synchronize()
        for n in NAMES:
            assert torch.equal(got[n], ref[n]), f"call {call}: {n}"
    assert F.fp8_device_error() == 0


def test_noalloc_route_rejects_problems_over_its_scratch(cuda_device):
    # (ceil(16384 * 8 / 512) + 1) * 256 int32 = 65792 > 65536
    scores = torch.zeros((16384, 256), dtype=torch.float32, device=cuda_device)
    with pytest.raises(F.Fp8Error) as err:
        F.moe_route_noalloc(scores, 8)
    assert err.value.code == 2          # FP8_ERR_SHAPE
