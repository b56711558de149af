"""A bounded device-side wait that runs out is reported, and the kernel returns.

The decoder resolves the thread boundaries of a chunk in fix-up rounds and
gives up after a round limit, reporting EH_ERR_TIMEOUT; consistent data never
reaches the default limit.  The test hook eh_debug_set_fixup_rounds lowers the
limit to one round, and a tensor of 1024-value chunks (windows of a few bits,
whose ends move in the first round) makes the decoder give up.  This is pure
computation: no wait on memory or another thread is cut short.  The status
word must read EH_ERR_TIMEOUT, the context must stay usable, and with the
default limit restored the same call must decode exactly.
"""
import numpy as np
import pytest
import torch

from exponent_entropy_coding_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def eh():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exponent_entropy_coding_b200 import build, exphuff
    build.build()
    exphuff.lib()
    return exphuff


def test_fixup_round_limit_reports_timeout(eh):
    x = synth.normal_bf16(200 * 1024 + 7, seed=11)
    t = torch.from_numpy(x.view(np.int16)).cuda()
    p = eh.plan(eh.EH_BF16, 1024)
    c = eh.compress(t, p)
    ws = torch.empty(eh.decompress_workspace(p, 1), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(t)
    try:
        eh.debug_set_fixup_rounds(1)
        eh.decompress(c, p, out=y, workspace=ws, check=False)
        assert eh.get_status(ws) == eh.EH_ERR_TIMEOUT
    finally:
        eh.debug_set_fixup_rounds(0)
    torch.cuda.synchronize()  # the kernel returned; the context is usable
    eh.decompress(c, p, out=y, workspace=ws)
    assert eh.get_status(ws) == eh.EH_OK
    assert torch.equal(y, t)
