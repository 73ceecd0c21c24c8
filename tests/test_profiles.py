"""The ncu summaries under profiles/ stay reproducible from committed files: every command
they record runs bench.py with flags and profile cases bench.py defines, every ncu command
leaves the clocks alone (--clock-control none), and each summary names its kernel."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _commands(text):
    """Commands inside fenced blocks, with backslash continuations joined."""
    out = []
    for block in re.findall(r"```\n(.*?)```", text, flags=re.S):
        joined = re.sub(r"\\\n\s*", " ", block)
        out += [line.strip() for line in joined.splitlines() if line.strip()]
    return out


def _bench_flags_and_cases():
    src = open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read()
    flags = set(re.findall(r'add_argument\("(--[a-z0-9-]+)"', src))
    cases = set(re.findall(r'"(gemv_\d+x\d+)": \(', src)) | set(re.findall(r'name == "([a-z0-9_]+)"', src))
    return flags, cases


def test_profile_commands_match_the_committed_bench():
    flags, cases = _bench_flags_and_cases()
    assert {"--steps", "--warmup", "--profile-case", "--no-e2e"} <= flags and cases
    files = sorted(f for f in os.listdir(os.path.join(ROOT, "profiles")) if f.endswith(".md"))
    assert files
    for f in files:
        text = open(os.path.join(ROOT, "profiles", f), encoding="utf-8").read()
        cmds = _commands(text)
        assert any(c.startswith("ncu ") for c in cmds), f
        for c in cmds:
            if c.startswith("ncu "):
                assert "--clock-control none" in c, (f, c)
            assert "python bench.py" in c, (f, c)
            args = c.split("python bench.py", 1)[1].split()
            for a in args:
                if a.startswith("--"):
                    assert a in flags, (f, a)
            if "--profile-case" in args:
                assert args[args.index("--profile-case") + 1] in cases, (f, c)
