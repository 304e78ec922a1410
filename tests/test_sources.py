"""Source invariants of the CUDA library that no GPU is needed to check.

Every kernel is launched with programmatic stream serialization, which lets it be scheduled
before the previous kernel on the stream has finished.  Stream order then rests on two rules:
every launch goes through the one launch helper, and every kernel waits for its predecessor
(griddep_wait, or griddep_enter which includes it) before touching global memory.  A kernel
added without the wait would read or overwrite data of a kernel still running.
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sample_gradient_clipping_b200", "csrc")


def _kernel_bodies():
    """(name, body) of every __global__ function in the CUDA sources."""
    out = []
    for fn in sorted(os.listdir(CSRC)):
        if not fn.endswith((".cu", ".cuh")):
            continue
        text = open(os.path.join(CSRC, fn)).read()
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"__global__", text):
            brace = text.index("{", m.end())
            depth, j = 0, brace
            while True:
                depth += {"{": 1, "}": -1}.get(text[j], 0)
                if depth == 0:
                    break
                j += 1
            head = text[m.end():brace]
            name = re.findall(r"([A-Za-z_][A-Za-z0-9_]*)\s*\(", head)
            name = [n for n in name if n != "__launch_bounds__" and n != "__cluster_dims__"][0]
            out.append((f"{fn}:{name}", text[brace + 1:j]))
    return out


def _device_body(name):
    """Text of the device function `name` (a kernel body shared by several entry points)."""
    for fn in sorted(os.listdir(CSRC)):
        if not fn.endswith((".cu", ".cuh")):
            continue
        text = re.sub(r"//[^\n]*", "", open(os.path.join(CSRC, fn)).read())
        m = re.search(r"__device__[^;{]*\b" + name + r"\s*\(", text)
        if m:
            brace = text.index("{", m.end())
            depth, j = 0, brace
            while True:
                depth += {"{": 1, "}": -1}.get(text[j], 0)
                if depth == 0:
                    return text[brace + 1:j]
                j += 1
    return ""


def test_every_kernel_waits_for_its_predecessor():
    bodies = _kernel_bodies()
    assert len(bodies) >= 18
    for name, body in bodies:
        # An entry point whose whole work is a shared body function: check that function.
        call = re.match(r"\s*([A-Za-z_][A-Za-z0-9_]*_body)\s*(<[^>]*>)?\s*\(", body)
        if call and not re.search(r"\bgriddep_(enter|wait)\(\)", body):
            body = _device_body(call.group(1))
        m = re.search(r"\bgriddep_(enter|wait)\(\)", body)
        assert m, f"{name} never waits for the previous kernel"
        before = body[:m.start()]
        # Before the wait only kernel-local work: no pointer parameters dereferenced, no
        # global loads or stores through the usual access forms, no device step read.
        assert "step.get()" not in before and "__ldg" not in before and "atomic" not in before, name


def test_every_launch_goes_through_the_helper():
    text = open(os.path.join(CSRC, "dpclip.cu")).read()
    text = re.sub(r"//[^\n]*", "", text)
    assert "<<<" not in text, "a kernel is launched without programmatic stream serialization"
    assert "cudaLaunchAttributeProgrammaticStreamSerialization" in text


def test_noise_tables_match_their_generator():
    """The committed Box-Muller tables are exactly what gen_noise_tables.py writes (mpmath at
    60 digits, each value rounded once), so the transform's constants cannot drift."""
    import importlib.util

    spec = importlib.util.spec_from_file_location("gen_noise_tables", os.path.join(CSRC, "gen_noise_tables.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    with open(os.path.join(CSRC, "noise_tables.cuh")) as f:
        assert f.read() == gen.render()


def _profile_commands():
    """(file, command) of every command in the fenced blocks of the ncu summaries in profiles/,
    continuation lines joined and `&&` chains split."""
    out = []
    pdir = os.path.join(ROOT, "profiles")
    for fn in sorted(os.listdir(pdir)):
        text = open(os.path.join(pdir, fn)).read()
        for block in re.findall(r"```[^\n]*\n(.*?)```", text, flags=re.S):
            joined = re.sub(r"\\\n\s*", " ", block)
            for line in joined.splitlines():
                for cmd in line.split("&&"):
                    if cmd.strip():
                        out.append((fn, cmd.strip()))
    return out


def test_profiles_hold_summaries_whose_commands_run_committed_files():
    """The ncu summaries are text, each gives the command that made it, every ncu command leaves
    the clocks alone, and every script it runs is part of the repository."""
    pdir = os.path.join(ROOT, "profiles")
    assert all(fn.endswith((".md", ".txt")) for fn in os.listdir(pdir))
    cmds = _profile_commands()
    files = {fn for fn, _ in cmds}
    assert files == {fn for fn in os.listdir(pdir)}, "a summary without its command"
    for fn, cmd in cmds:
        if cmd.startswith("ncu "):
            assert "--clock-control none" in cmd, (fn, cmd)
        for script in re.findall(r"\bpython\s+(?:-m\s+([\w.]+)|([\w./]+\.py))", cmd):
            mod, path = script
            target = os.path.join(ROOT, *mod.split(".")) + ".py" if mod else os.path.join(ROOT, path)
            assert os.path.exists(target), (fn, cmd)
