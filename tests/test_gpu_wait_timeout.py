"""The failure path of a bounded device wait, exercised without faulting or
hanging the GPU.

Every wait inside the decode kernels polls its mbarrier against a wall-clock
bound.  The test shortens that bound to 1 ms and switches on the library's test
hook that makes each CTA's copy producer stop issuing state copies from its
second half-tile on, so the consumers' wait for that half-tile can only run
out.  The kernel must record the timeout in the device error word, stop
releasing and refilling its shared-memory buffers, wait for the bulk copies it
already issued, and return.  The test then checks that the error is reported
(and cleared by reading), and that the same context still computes a correct
decode step afterwards (compared with the float64 oracle).  Both launch forms
are covered: 64 rows on the persistent grid, and 2 rows whose q/k groups run
as clusters of 3 CTAs (where the group's first CTA also waits for its peers'
signals before it exits).
"""
import numpy as np
import pytest
import torch

import gated_deltanet_mixer_gdn_b200 as gdn
from gated_deltanet_mixer_gdn_b200 import synth

from _util import check_outputs, oracle_prefill, to_dev

pytestmark = pytest.mark.gpu

GDN_DEVERR_TIMEOUT_COPY = 1


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    gdn.load_library()


@pytest.mark.parametrize("rows", [64, 2])
def test_decode_wait_runs_out_reports_and_returns(rows):
    case = synth.decode_case(4400 + rows, rows=rows, steps=1)
    w, _, st0, cv0 = to_dev(case)
    acts = [case[k][0].cuda() for k in ("qkv", "z", "a", "b")]
    assert gdn.last_device_error() == 0
    st, cv = st0.clone(), cv0.clone()
    lib = gdn.load_library()
    gdn.set_decode_wait_limit(1_000_000)
    assert lib.gdn_test_decode_stop_copies_at(1) == 0
    try:
        gdn.decode(*acts, w, st, cv)
        torch.cuda.synchronize()
    finally:
        assert lib.gdn_test_decode_stop_copies_at(-1) == 0
        gdn.set_decode_wait_limit()
    assert gdn.last_device_error() == GDN_DEVERR_TIMEOUT_COPY
    assert gdn.last_device_error() == 0  # cleared by the read

    # the context is usable: one step from the original state matches the oracle
    st, cv = st0.clone(), cv0.clone()
    out = gdn.decode(*acts, w, st, cv)
    torch.cuda.synchronize()
    ref = oracle_prefill(case, cu=np.arange(rows + 1), acts={k: case[k][0] for k in ("qkv", "z", "a", "b")})
    check_outputs(f"decode after a timed-out call ({rows} rows)", out, ref["out"], st, ref["state"], cv,
                  ref["conv"])
    assert gdn.last_device_error() == 0
