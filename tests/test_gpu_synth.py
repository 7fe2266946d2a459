"""The device table filler reproduces the host generator bit for bit (input generation)."""
import numpy as np
import pytest
import torch

from synth import device as sdev
from synth import gen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_device_fill_matches_host_generator(dtype):
    rows, width = 3001, 520
    t = torch.empty((rows, width), dtype=dtype, device="cuda")
    sdev.fill_table(t, 7, gen.TAG_SUBTABLE0 + 2, 0.02)
    pick = np.array([0, 1, 999, 3000, 1234])
    if dtype == torch.bfloat16:
        got = t[torch.from_numpy(pick).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
        want = gen.table_rows_bf16(7, gen.TAG_SUBTABLE0 + 2, pick, width, 0.02)
    else:
        got = t[torch.from_numpy(pick).cuda()].cpu().numpy()
        want = gen.table_values_f32(7, gen.TAG_SUBTABLE0 + 2, pick, width, 0.02)
    np.testing.assert_array_equal(got, want)
