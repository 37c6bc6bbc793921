"""The ncu raw-CSV reader behind profiles/traffic.json (CPU, synthetic CSV)."""

import csv

from fourier_neural_spectral_fno_b200 import profile_traffic as PT


def _write(path, rows):
    with open(path, "w", newline="") as f:
        csv.writer(f).writerows(rows)


def test_parse_scales_each_column_by_its_own_unit_and_averages(tmp_path):
    hdr = ["ID", "Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum"]
    units = ["", "", "Mbyte", "Kbyte"]
    rows = [hdr, units,
            ["0", "void fno::<unnamed>::k_epi_pipe<float, 1, 32>(CUtensorMap_st, ...)", "150", "80"],
            ["1", "void fno::<unnamed>::k_epi_pipe<float, 1, 32>(CUtensorMap_st, ...)", "152", "82"],
            ["2", "void fno::<unnamed>::k_epilogue<__nv_bfloat16, 3, 64, 128>(EpiArgs, Geom)",
             "1000", "300"],
            ["3", "void fno::<unnamed>::k_proj_bwd<__nv_bfloat16, 64>(const T1 *, ...)", "10",
             "n/a"],
            ["4", "void at::native::vectorized_elementwise_kernel<4>(...)", "5", "5"]]
    path = tmp_path / "raw.csv"
    _write(path, rows)
    acc = PT.parse(str(path))
    rd, wr, n = acc[("epi_block_fwd_pipe", "epilogue_pipe.cu")]
    assert n == 2
    assert rd / n == 151e6 and wr / n == 81e3
    rd, wr, n = acc[("epi_block_bwd", "epilogue.cu")]
    assert (rd, wr, n) == (1000e6, 300e3, 1)
    assert ("proj_bwd", "net.cu") not in acc            # unparsable value skipped
    assert len(acc) == 2                               # torch kernels ignored


def test_kernel_keys():
    assert PT._kernel_key("void fno::<unnamed>::k_epilogue<float, 1, 32, 256>(EpiArgs, Geom)") \
        == ("epi_block_fwd", "epilogue.cu")
    assert PT._kernel_key("k_lift4<float>(const float *)") == ("lift", "net.cu")
    assert PT._kernel_key("k_unknown(int)") is None
