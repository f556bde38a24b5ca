"""The committed ncu summaries: every capture command keeps the GPU's clocks
as they are (``--clock-control none``), and runs committed files only."""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _commands(text):
    """ncu command lines (continuations joined) from a summary's text."""
    out, cur = [], None
    for raw in text.splitlines():
        line = raw.strip().lstrip("#").strip()
        if cur is None and line.startswith("ncu --"):
            cur = ""
        if cur is not None:
            cur += " " + line.rstrip("\\").strip()
            if not line.endswith("\\"):
                out.append(cur.strip())
                cur = None
    return out


def test_every_capture_keeps_the_clocks_and_runs_committed_files():
    files = sorted(glob.glob(os.path.join(ROOT, "profiles", "*")))
    assert files
    n = 0
    for path in files:
        assert path.endswith((".md", ".txt")), f"{path}: summaries only"
        assert os.path.getsize(path) < 16 * 1024, f"{path}: keep summaries short"
        for cmd in _commands(open(path).read()):
            n += 1
            assert "--clock-control none" in cmd, f"{os.path.basename(path)}: {cmd}"
            for script in re.findall(r"python\s+(\S+\.py)", cmd):
                assert os.path.exists(os.path.join(ROOT, script)), f"{os.path.basename(path)}: {script}"
                assert not script.startswith("_work"), f"{os.path.basename(path)}: {script}"
    assert n >= 8
