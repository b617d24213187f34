"""The gather probe on the GPU: the shared-memory layout it reads back is the one it
lands, for every loader and both row sizes, no wait times out, and the rates it reports
are plausible.  The probe supplies the SM-side roofline of the benchmark (the rate at which
random rows of an L2-resident buffer reach shared memory and are read back), so its
layouts and its completion are checked here rather than trusted."""
from __future__ import annotations

import pytest
import torch

import top_sparse_attention_index_b200 as qsa
from top_sparse_attention_index_b200 import gather_probe

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("row_bytes", [512, 256])
@pytest.mark.parametrize("method", [0, 1, 2, 3])
def test_probe_layout_check(cuda_device, method, row_bytes):
    """read_back 2: every fragment read back is compared with the source bytes of its row."""
    buf = torch.randint(-2**31, 2**31 - 1, ((8 << 20) // 4,), dtype=torch.int32,
                        device=cuda_device, generator=torch.Generator(device=cuda_device).manual_seed(5))
    sink = torch.zeros(258, dtype=torch.int32, device=cuda_device)
    rows = (8 << 20) // row_bytes
    stream = torch.cuda.current_stream(cuda_device)
    st = qsa.qsa_probe_gather(method, 2, buf.data_ptr(), rows, row_bytes, row_bytes, 4, 2, 16, 8,
                              7, sink.data_ptr(), stream.cuda_stream)
    assert st == qsa.QSA_OK, qsa.qsa_last_error_detail()
    torch.cuda.synchronize()
    assert int(sink[0]) == 0, "a wait timed out or the shared memory was misaligned"
    assert int(sink[1]) == 0, "fragments read back differ from the rows gathered"


def test_probe_pitch_and_strided_rows(cuda_device):
    """Rows 1,024 bytes apart (a 512-byte row of each slot of a [S, 2, 256] bf16 cache):
    the layout check holds with a pitch larger than the row."""
    buf = torch.randint(-2**31, 2**31 - 1, ((16 << 20) // 4,), dtype=torch.int32,
                        device=cuda_device, generator=torch.Generator(device=cuda_device).manual_seed(6))
    sink = torch.zeros(258, dtype=torch.int32, device=cuda_device)
    stream = torch.cuda.current_stream(cuda_device)
    for method in (0, 1):
        st = qsa.qsa_probe_gather(method, 2, buf.data_ptr(), (16 << 20) // 1024, 1024, 512, 4, 3,
                                  8, 6, 11, sink.data_ptr(), stream.cuda_stream)
        assert st == qsa.QSA_OK, qsa.qsa_last_error_detail()
    torch.cuda.synchronize()
    assert int(sink[0]) == 0 and int(sink[1]) == 0


def test_gather_peak_is_plausible(cuda_device):
    """The benchmark's peak: the best of the probe's runs, finite, every run completed,
    and below what the SMs' L1 could take in at all (a few hundred bytes per SM clock)."""
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    r = gather_probe.gather_peak(cuda_device, 512, reps=2)
    assert all(x["tb_per_s"] is not None for x in r["runs"])
    assert r["tb_per_s"] == max(x["tb_per_s"] for x in r["runs"])
    assert 1.0 < r["tb_per_s"] < sms * 256 * 2.1e9 / 1e12


def test_mma_operand_probe(cuda_device):
    """The MMA operand-rate probe: every tcgen05 accumulator element comes out exact, no
    wait times out, and the rates are positive; the tensor core's MAC rate at N = 256 is
    the order of the dense peak (one MMA of 128 x 256 x 16 per ~128 cycles or better)."""
    from top_sparse_attention_index_b200.gather_probe import MMA_N, mma_operand_rates
    r = mma_operand_rates(cuda_device, rounds=200)
    assert r["ldmatrix_x4_16_warps"]["timeouts"] == 0
    assert r["ldmatrix_x4_16_warps"]["bytes_per_clk_per_sm"] > 0
    for n in MMA_N:
        d = r["tcgen05"][str(n)]
        assert d["timeouts"] == 0 and d["mismatches"] == 0, (n, d)
        assert d["bytes_per_clk_per_sm"] > 0
    assert r["tcgen05"]["256"]["mac_per_clk_per_sm"] > 1000
