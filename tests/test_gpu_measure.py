"""The measurement entry point amk_read_ceiling on the device: the decode
kernel's bulk-copy weight stream with nothing consuming it must read at an
HBM-like rate (well above the CPU's, not above the part's 8 TB/s) and stop
cleanly."""
import pytest
import torch

import persistent_megakernel_decode_cta_b200 as amk
from persistent_megakernel_decode_cta_b200 import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    build.build()


def test_read_ceiling_is_an_hbm_rate():
    buf = torch.ones(1 << 30, dtype=torch.uint8, device="cuda")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    g = amk.read_ceiling(buf, sms, 32768, 3, reps=2)
    assert 2000.0 < g < 9000.0, g
    del buf
    torch.cuda.empty_cache()
