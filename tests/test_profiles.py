"""The commands quoted in profiles/ run committed files only and keep the
profiling rules: every ncu command carries --clock-control none, every
bench.py command line parses with bench.py's own parser, and every pytest
target exists.  A single capital letter in a command stands for a number
(the summary's table gives its values)."""
import glob
import os
import re
import shlex

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUMMARIES = sorted(glob.glob(os.path.join(ROOT, "profiles", "*")))


def logical_lines(path):
    text = open(path).read()
    text = re.sub(r"\\\n\s*", " ", text)          # shell line continuations
    text = re.sub(r"\]\n\s*", "] ", text)          # an option list broken over lines
    return text.splitlines()


def command_spans(line, word, anywhere=False):
    """The commands on a line that start with ``word``: the text from it up to
    a closing backtick or the end of the line.  Unless ``anywhere``, only where
    a command can start (the line's start, after "# command:", a backtick or
    "&&"), so that a heading naming a tool ("(ncu --set full)") is not taken
    for a command; a program run under ncu is found with ``anywhere``."""
    start = "" if anywhere else r"(?:^\s*(?:# command:\s*)?|`|&&\s*)"
    return [m.group(1) for m in re.finditer(start + "(" + re.escape(word) + r"[^`]*)", line)]


def numbers_for_placeholders(args):
    return ["1" if re.fullmatch(r"[A-Z]", a) else a for a in args
            if not (a.startswith("[") or a.endswith("]"))]


def test_there_are_summaries():
    assert SUMMARIES and all(p.endswith((".md", ".txt")) for p in SUMMARIES)


@pytest.mark.parametrize("path", SUMMARIES, ids=os.path.basename)
def test_every_ncu_command_leaves_the_clocks_alone(path):
    found = False
    for line in logical_lines(path):
        for cmd in command_spans(line, "ncu --"):
            found = True
            assert "--clock-control none" in cmd, (path, cmd)
    assert found, f"{path} quotes no ncu command"


@pytest.mark.parametrize("path", SUMMARIES, ids=os.path.basename)
def test_bench_and_pytest_commands_use_committed_files(path):
    parser = bench.build_parser()
    for line in logical_lines(path):
        assert "_work/" not in line, (path, line)
        for cmd in command_spans(line, "python bench.py", anywhere=True):
            args = numbers_for_placeholders(shlex.split(cmd)[2:])
            parser.parse_args(args)                     # exits on an unknown option
        for cmd in command_spans(line, "python -m pytest ", anywhere=True):
            words = shlex.split(cmd)[3:]
            files = [w for w in words if w.endswith(".py")]
            assert files, (path, cmd)
            for f in files:
                assert os.path.exists(os.path.join(ROOT, f)), (path, f)
            if "-k" in words:
                name = words[words.index("-k") + 1]
                src = "".join(open(os.path.join(ROOT, f)).read() for f in files)
                assert re.search(r"def test_\w*" + re.escape(name), src), (path, name)
