"""Host-side helpers of bench.py (CPU only): the code-only source hash that ties a recorded DRAM-traffic figure
to the kernel source it was captured on."""
import bench


SRC = """// header comment
#include <x.h>
/* block
   comment */
__global__ void k(int* p) {  // trailing comment
    p[0] = 1;

}
"""


def test_code_only_drops_comments_and_blank_lines():
    assert bench._code_only(SRC) == "#include <x.h>\n__global__ void k(int* p) {\n    p[0] = 1;\n}"


def test_comment_edit_keeps_the_code_and_a_code_edit_changes_it():
    reworded = SRC.replace("// trailing comment", "// another wording").replace("header comment", "new header")
    assert bench._code_only(reworded) == bench._code_only(SRC)
    assert bench._code_only(SRC.replace("p[0] = 1;", "p[0] = 2;")) != bench._code_only(SRC)


def test_recorded_traffic_needs_the_recorded_code(tmp_path, monkeypatch):
    """A record whose hash is not the current code's gives no traffic figure (null in the JSON line)."""
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text(SRC)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash("k.cu")
    (tmp_path / "profiles" / "traffic.json").write_text(
        '{"k@w": {"dram_bytes_per_launch": 123, "source_hash": "%s"}, "k@v": {"dram_bytes_per_launch": 1, '
        '"source_hash": "0000000000000000"}}' % h)
    assert bench.recorded_traffic("k", "w", ("k.cu",)) == 123.0
    assert bench.recorded_traffic("k", "v", ("k.cu",)) is None
    assert bench.recorded_traffic("k", "missing", ("k.cu",)) is None
