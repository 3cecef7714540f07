"""The read-bandwidth probe (the L2 term of the decode roofline) reads what it
is given and reports its pass count; buffer sizes that are not a whole number
of its 8-load batches exercise the tail loop."""
import pytest
import torch

import weight_shared_looped_b200 as tl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbytes", [16, 4096 + 16, 32 << 20])
@pytest.mark.parametrize("passes", [1, 3])
def test_read_probe_runs_and_reports_passes(nbytes, passes):
    buf = torch.ones(nbytes, dtype=torch.uint8, device="cuda")
    sink = torch.zeros(2, dtype=torch.int32, device="cuda")
    tl.tl_read_probe(buf, passes, sink)
    torch.cuda.synchronize()
    assert int(sink[1].item()) == passes
    assert int(sink[0].item()) == 0          # the fold of all-ones words never hits the marker
