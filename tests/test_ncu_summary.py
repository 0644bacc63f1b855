"""The profile summariser on a small synthetic ncu CSV (host logic, CPU)."""
from token_recurrent_decoding_b200 import ncu_summary

HDR = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream",'
       '"Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit",'
       '"Metric Value"\n')


def row(i, name, ns):
    return (f'"{i}","1","python","h","{name}","1","7","(128, 1, 1)","(1, 1, 1)","0","10.0",'
            f'"Command line profiler metrics","gpu__time_duration.sum","nsecond","{ns}"\n')


def test_launch_list_groups_by_kernel_and_shares(tmp_path):
    p = tmp_path / "launches.csv"
    p.write_text("==PROF== noise before the table\n" + HDR
                 + row(0, "void rlt::k_a<64, 2>(int, const float *)", "1,000")
                 + row(1, "void rlt::k_a<64, 2>(int, const float *)", "3000")
                 + row(2, "rlt::k_b(float *)", "4000")
                 + row(3, "void at::other_kernel<float>(int)", "2000"))
    out = ncu_summary.launches(str(p), match="rlt::").splitlines()
    rows = {l.split()[0]: l.split() for l in out[1:-1]}
    # template arguments kept, parameter lists dropped; shares of the listed time
    assert rows["rlt::k_a<64,"][-4:] == ["2", "4.0", "2.00", "0.500"]
    assert rows["rlt::k_b"][-4:] == ["1", "4.0", "4.00", "0.500"]
    assert out[-1].split()[-2:] == ["3", "8.0"]


def test_kernel_key():
    assert ncu_summary.kernel_key("void rlt::f<a<1>, 2>(int, b<3>)") == "rlt::f<a<1>, 2>"
    assert ncu_summary.kernel_key("k(int)") == "k"
