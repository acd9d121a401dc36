"""The dense prefill's schedule as the library reports it (gdn_prefill_segments):
overlap only where the recurrence leaves SMs free and the rows are long enough,
and segment counts within the library's bound."""
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    gdn.load_library()


def test_segments():
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    assert gdn.prefill_segments(0, 100) == 0
    assert gdn.prefill_segments(1, 0) == 0
    assert gdn.prefill_segments(1, 15 * 64) == 1          # under 16 chunks: plain schedule
    s1 = gdn.prefill_segments(1, 8192)
    assert 2 <= s1 <= 8                                  # one row: the recurrence leaves SMs free
    s2 = gdn.prefill_segments(2, 65536)
    assert 2 <= s2 <= 8
    rows = (nsm - 32) // 48 + 1                          # the recurrence would take too many SMs
    assert gdn.prefill_segments(rows, 8192) == 1
    with pytest.raises(gdn.GdnError):
        gdn.prefill_segments(-1, 8)
