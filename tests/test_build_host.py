"""The in-tree build: stale sources compile in parallel; a source that fails
to compile raises with the compiler's output and leaves no object behind that
a later build would take for up to date."""
import os

import pytest

from w4a4_diffusion_transformer_b200 import build


def test_a_failing_source_raises_and_leaves_no_object(tmp_path, monkeypatch):
    csrc = tmp_path / "csrc"
    csrc.mkdir()
    (csrc / "good.cpp").write_text("int good() { return 1; }\n")
    (csrc / "bad.cpp").write_text("int bad( { return ; }\n")
    monkeypatch.setattr(build, "CSRC", str(csrc))
    monkeypatch.setattr(build, "BUILD", str(tmp_path / "_build"))
    monkeypatch.setattr(build, "LIB", str(tmp_path / "lib.so"))
    monkeypatch.setattr(build, "CUDA_SOURCES", [])
    monkeypatch.setattr(build, "CXX_SOURCES", ["good.cpp", "bad.cpp"])
    with pytest.raises(RuntimeError) as e:
        build.build()
    assert "bad.cpp" in str(e.value)
    objs = sorted(os.listdir(tmp_path / "_build"))
    assert "good.cpp.o" in objs                                   # the other job finished
    assert not any(o.startswith("bad.cpp.o") and not o.endswith(".tmp") for o in objs)
    assert not (tmp_path / "lib.so").exists()
    # once fixed, the next build compiles only what is stale and links
    (csrc / "bad.cpp").write_text("int bad() { return 0; }\n")
    assert build.build() == str(tmp_path / "lib.so")
    assert (tmp_path / "lib.so").exists()
