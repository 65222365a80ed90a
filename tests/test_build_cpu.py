"""The build's tuning-define hook (no GPU): MOE_BUILD_DEFINES parsing and the
stamp comparison that decides whether the library on disk is up to date."""
import pytest

from moe_expert_epilogue_b200 import build


def test_defines_parsed_sorted_and_validated(monkeypatch):
    monkeypatch.setenv("MOE_BUILD_DEFINES", "MOE_RES_WIDE=0  MOE_ACT_FLAT_CTAS=3")
    assert build.defines() == ["MOE_ACT_FLAT_CTAS=3", "MOE_RES_WIDE=0"]
    monkeypatch.setenv("MOE_BUILD_DEFINES", "MOE_PDL_TRIGGER")
    assert build.defines() == ["MOE_PDL_TRIGGER"]
    for bad in ("NOT_MOE=1", "MOE_X=1;rm", "MOE_X=abc", "MOE_X$=1"):
        monkeypatch.setenv("MOE_BUILD_DEFINES", bad)
        with pytest.raises(ValueError):
            build.defines()
    monkeypatch.delenv("MOE_BUILD_DEFINES")
    assert build.defines() == []


def test_stamp_must_match_the_requested_defines(monkeypatch, tmp_path):
    stamp = tmp_path / "lib.defines"
    monkeypatch.setattr(build, "STAMP", str(stamp))
    monkeypatch.delenv("MOE_BUILD_DEFINES", raising=False)
    assert build.built_defines() == []                 # no stamp: a default build
    stamp.write_text("MOE_PDL_TRIGGER=1")
    assert build.built_defines() == ["MOE_PDL_TRIGGER=1"]
    monkeypatch.setenv("MOE_BUILD_DEFINES", "MOE_PDL_TRIGGER=1")
    assert build.built_defines() == build.defines()
    monkeypatch.delenv("MOE_BUILD_DEFINES")
    assert build.built_defines() != build.defines()    # a plain run must rebuild
