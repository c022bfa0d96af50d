"""Lint of the committed ncu summaries (profiles/*.md), on the CPU: each names the
build it came from and the full command that made it; every ncu command leaves the
GPU clocks alone (--clock-control none), captures a bounded number of launches (-c),
and runs only committed entry points of this repository (bench.py or a module of
the package) with arguments they accept."""
import os
import re
import shlex

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = sorted(f for f in os.listdir(os.path.join(ROOT, "profiles")) if f.endswith(".md"))


def _commands(text):
    blocks = re.findall(r"```\n(.*?)```", text, flags=re.S)
    return [b.replace("\\\n", " ") for b in blocks if "ncu" in b]


def test_there_are_summaries():
    assert PROFILES


@pytest.mark.parametrize("name", PROFILES)
def test_summary_names_build_and_a_safe_command(name):
    text = open(os.path.join(ROOT, "profiles", name)).read()
    assert re.search(r"[Bb]uild: commit [0-9a-f]{7}", text), f"{name}: no build commit"
    cmds = _commands(text)
    assert cmds, f"{name}: no ncu command"
    for cmd in cmds:
        args = shlex.split(cmd)
        assert args[0] == "ncu"
        assert "--clock-control" in args and args[args.index("--clock-control") + 1] == "none", cmd
        assert "-c" in args and int(args[args.index("-c") + 1]) <= 400, cmd
        py = args.index("python")
        target = args[py + 1:]
        if target[0] == "-m":
            mod = target[1]
            assert mod.startswith("dynamic_short_convolutions_b200."), cmd
            path = os.path.join(ROOT, *mod.split(".")) + ".py"
        else:
            path = os.path.join(ROOT, target[0])
        assert os.path.exists(path), f"{name}: {path} is not in the repository"
        assert "_work" not in cmd and "/root/" not in cmd, cmd


@pytest.mark.parametrize("name", PROFILES)
def test_summary_command_arguments_are_accepted(name):
    """The profiled program's own argument parser takes the summary's arguments."""
    import importlib
    import sys

    text = open(os.path.join(ROOT, "profiles", name)).read()
    for cmd in _commands(text):
        args = shlex.split(cmd)
        target = args[args.index("python") + 1:]
        if target[0] == "-m":
            mod, rest = target[1], target[2:]
        else:
            mod, rest = os.path.splitext(target[0])[0], target[1:]
        sys.path.insert(0, ROOT)
        try:
            m = importlib.import_module(mod)
        finally:
            sys.path.pop(0)
        parser = m.build_parser() if hasattr(m, "build_parser") else None
        if parser is None:
            pytest.skip(f"{mod} exposes no build_parser()")
        ns = parser.parse_args(rest)
        if getattr(ns, "config", None) is not None:
            from dynamic_short_convolutions_b200 import workloads as W

            assert ns.config in W.CONFIGS, f"{name}: unknown workload {ns.config}"
