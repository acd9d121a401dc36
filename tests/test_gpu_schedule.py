"""The dense prefill's schedule as the library reports it (gdn_prefill_schedule):
overlap only where the recurrence leaves SMs free and the rows are long enough,
segment counts within the library's bound, launch counts consistent with them."""
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    gdn.load_library()


def test_schedule():
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    assert gdn.prefill_schedule(0, 100) == (0, 0)
    assert gdn.prefill_schedule(1, 0) == (0, 0)
    assert gdn.prefill_schedule(1, 15 * 64) == (1, 4)          # under 16 chunks: plain schedule
    assert gdn.prefill_schedule(1, 15 * 64, True) == (1, 4)    # fused in_proj GEMM, history, WY, recurrence
    assert gdn.prefill_schedule(1, 2, True) == (1, 4)          # short rows fuse too
    s1, l1 = gdn.prefill_schedule(1, 8192)
    assert 2 <= s1 <= 8 and l1 == 2 + 2 * s1
    s2, l2 = gdn.prefill_schedule(1, 8192, True)
    assert 2 <= s2 <= 8 and l2 == 2 + 2 * s2
    s3, l3 = gdn.prefill_schedule(2, 65536)
    assert 2 <= s3 <= 8 and l3 == 2 + 2 * s3
    rows = (nsm - 32) // 48 + 1                                # the recurrence would take too many SMs
    assert gdn.prefill_schedule(rows, 8192) == (1, 4)
    with pytest.raises(gdn.GdnError):
        gdn.prefill_schedule(-1, 8)
