"""Device-side error reporting: a bounded wait that runs out records
ROM_ERR_TIMEOUT in the status word and the context stays usable. The wait is
on an mbarrier that nothing arrives on, with a 2 ms limit; nothing faults or
hangs."""
import numpy as np
import pytest
import torch

from mixture_experts_projections_b200 import rom
from mixture_experts_projections_b200.inputs import make_block_inputs
from oracle import rom_oracle as orc
from parity_util import to_dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert rom.rom_get_status() == rom.ROM_OK
    rom.rom_debug_wait_timeout(2_000_000)
    assert rom.rom_get_status() == rom.ROM_ERR_TIMEOUT
    assert rom.rom_get_status() == rom.ROM_OK  # reading resets the word
    inp = make_block_inputs(300, 128, 1, 8, seed=4)
    bufs = rom.route_and_dispatch(to_dev(inp["x"], "bf16"), to_dev(inp["w_r"], "f32"), None, 8, 1,
                                  False)
    torch.cuda.synchronize()
    rt = orc.route(inp["x"], inp["w_r"], 1)
    assert np.array_equal(bufs.topk_idx.cpu().numpy(), rt["topk_idx"])


def test_invalid_arguments_raise_before_launch():
    x = torch.zeros((10, 12), dtype=torch.bfloat16, device="cuda")  # Dm % 8 != 0
    w_r = torch.zeros((12, 4), dtype=torch.float32, device="cuda")
    bufs = rom.RoutingBuffers(10, 12, 4, 1, torch.bfloat16, "cuda")
    with pytest.raises(rom.RomError, match="UNSUPPORTED"):
        rom.rom_route(x, w_r, None, 1, False, bufs.topk_idx, bufs.topk_w, None, bufs.ws)
    with pytest.raises(rom.RomError, match="INVALID_ARG"):
        rom.rom_route(x, w_r, None, 5, False, bufs.topk_idx, bufs.topk_w, None, bufs.ws)
