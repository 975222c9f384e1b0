"""The committed profile summaries: text only, and every command in them re-runnable from
committed files with the profiler's clock control off."""

import os
import re
import shlex
import sys

import pytest

from tests.conftest import ROOT

PROFILES = os.path.join(ROOT, "profiles")


def _commands(text):
    """Indented command lines of a summary, continuation lines joined."""
    cmds, cur = [], ""
    for line in text.splitlines():
        if not line.startswith("    "):
            if cur:
                cmds.append(cur)
            cur = ""
            continue
        part = line.strip()
        cur = (cur + " " + part) if cur else part
        if not part.endswith("\\"):
            cmds.append(cur)
            cur = ""
    if cur:
        cmds.append(cur)
    return [c.replace("\\ ", " ") for c in cmds]


def test_profiles_hold_text_summaries_only():
    names = os.listdir(PROFILES)
    assert names
    for n in names:
        assert n.endswith((".md", ".txt")), n
        assert os.path.getsize(os.path.join(PROFILES, n)) < 64 * 1024, n


def test_profile_commands_run_committed_files_with_clock_control_off():
    seen_ncu = 0
    for n in sorted(os.listdir(PROFILES)):
        if not n.endswith(".md"):
            continue
        with open(os.path.join(PROFILES, n)) as f:
            text = f.read()
        for cmd in _commands(text):
            if re.search(r"(^|\s)ncu\s", cmd):
                seen_ncu += 1
                assert "--clock-control none" in cmd, f"{n}: {cmd}"
            for script in re.findall(r"python\s+(\S+\.py)", cmd):
                assert not script.startswith("_work"), f"{n}: {cmd}"
                assert os.path.isfile(os.path.join(ROOT, script)), f"{n}: {script} is not in the repository"
    assert seen_ncu > 0


def test_profile_bench_commands_parse_with_the_current_bench(monkeypatch):
    """Every bench.py command line in the summaries is accepted by bench.py's argument parser."""
    sys.path.insert(0, ROOT)
    import bench
    checked = 0
    for n in sorted(os.listdir(PROFILES)):
        if not n.endswith(".md"):
            continue
        with open(os.path.join(PROFILES, n)) as f:
            text = f.read()
        for cmd in _commands(text):
            words = shlex.split(cmd)
            for i, w in enumerate(words[:-1]):
                if w == "python" and words[i + 1] == "bench.py":
                    monkeypatch.setattr(sys, "argv", words[i + 1:])
                    try:
                        bench.parse()
                    except SystemExit:
                        pytest.fail(f"{n}: bench.py rejects {' '.join(words[i + 1:])}")
                    checked += 1
    assert checked > 0
