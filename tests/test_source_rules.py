"""Rules of the GPU code that can be checked on the sources, without a GPU:
every mbarrier poll goes through the one bounded wait, every file that
allocates tensor memory also frees it, and every ncu command recorded under
profiles/ leaves the GPU clocks alone."""
import pathlib
import re

ROOT = pathlib.Path(__file__).resolve().parents[1]
CSRC = ROOT / "paged_kv_cache_459_b200" / "csrc"
SOURCES = sorted(p for p in CSRC.iterdir() if p.suffix in (".cu", ".cuh", ".h", ".cpp"))


def _code(path: pathlib.Path) -> str:
    """The file without // and /* */ comments."""
    text = path.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def _call_args(code: str, start: int) -> list[str]:
    """Top-level arguments of the call whose '(' ends just before `start`."""
    depth, args, cur = 1, [], []
    for ch in code[start:]:
        if ch in "([{":
            depth += 1
        elif ch in ")]}":
            depth -= 1
            if depth == 0:
                args.append("".join(cur).strip())
                return args
        if ch == "," and depth == 1:
            args.append("".join(cur).strip())
            cur = []
        else:
            cur.append(ch)
    raise AssertionError("unbalanced call")


def test_sources_found():
    names = {p.name for p in SOURCES}
    assert {"ptx.cuh", "decode_unit.cuh", "prefill_tc.cu", "decode_prefix.cu"} <= names


def test_mbarrier_polls_go_through_the_bounded_wait():
    """Only ptx.cuh polls an mbarrier (one poll at CTA scope, one acquiring at
    cluster scope), and each of its two loops gives up after a globaltimer
    limit; every other file waits through mbar_wait(bar, parity, limit) or
    mbar_wait_cluster(bar, parity, limit)."""
    for path in SOURCES:
        code = _code(path)
        if path.name == "ptx.cuh":
            assert code.count("mbarrier.try_wait") == 2
            loops = re.findall(r"while\s*\(\s*true\s*\)|for\s*\(\s*;\s*;\s*\)", code)
            assert len(loops) == 2
            for name in ("bool mbar_wait(", "bool mbar_wait_cluster("):
                body = code[code.index(name):]
                body = body[:body.index("\n}\n")]
                assert "globaltimer_ns() - t0 > limit_ns" in body and "return false" in body, name
            continue
        assert "mbarrier.try_wait" not in code and "mbarrier.wait" not in code, path.name
        assert "mbar_try_wait(" not in code and "mbar_try_wait_cluster(" not in code, path.name
        for m in re.finditer(r"\bmbar_wait(_cluster)?\(", code):
            args = _call_args(code, m.end())
            assert len(args) == 3 and args[2], f"{path.name}: mbarrier wait without a limit: {args}"


def test_no_unbounded_spin_loops_in_kernels():
    for path in SOURCES:
        if path.name == "ptx.cuh":
            continue
        code = _code(path)
        assert not re.search(r"while\s*\(\s*(true|1)\s*\)", code), path.name
        # the one "for (;;)" form allowed is a walk over a finite item list that returns
        for m in re.finditer(r"for\s*\(\s*;\s*;", code):
            tail = code[m.end():m.end() + 600]
            assert "return" in tail or "break" in tail, f"{path.name}: endless loop"


def test_tensor_memory_is_freed_where_it_is_allocated():
    for path in SOURCES:
        code = _code(path)
        allocs = len(re.findall(r"tcgen05\.alloc\.|tc::alloc<", code))
        deallocs = len(re.findall(r"tcgen05\.dealloc\.|tc::dealloc<", code))
        if path.name == "tcgen05.cuh":  # the helpers themselves
            assert allocs == 1 and deallocs == 1
            continue
        assert allocs == deallocs, f"{path.name}: {allocs} allocations, {deallocs} frees"


def test_recorded_ncu_commands_leave_the_clocks_alone():
    found = 0
    for md in sorted((ROOT / "profiles").glob("*.md")):
        # join backslash-continued lines into one command line
        text = md.read_text().replace("\\\n", " ")
        for line in text.splitlines():
            if re.search(r"(^|[\s;&|(])ncu\s", line):
                found += 1
                assert "--clock-control none" in line, f"{md.name}: {line.strip()}"
    assert found > 0


def test_every_environment_switch_is_documented():
    """Each environment variable the library reads is described in the public
    header (the kernels it selects, their defaults)."""
    header = (ROOT / "include" / "pkv.h").read_text()
    names = set()
    for path in SOURCES:
        names |= set(re.findall(r'(?:env_int|getenv)\(\s*"([A-Z0-9_]+)"', _code(path)))
    assert names, "no environment switch found"
    missing = sorted(n for n in names if n not in header)
    assert not missing, missing


def _imports(path: pathlib.Path) -> set[str]:
    """Top-level names of the modules a Python file imports."""
    names = set()
    for m in re.finditer(r"^\s*(?:from\s+([\w.]+)\s+import|import\s+([\w., ]+))", path.read_text(),
                         flags=re.M):
        if m.group(1):
            names.add(m.group(1).split(".")[0])
        else:
            names |= {n.strip().split(" ")[0].split(".")[0] for n in m.group(2).split(",")}
    return names


def test_oracle_side_never_imports_the_library():
    """The oracle and its pins share no code with the CUDA path: nothing under
    oracle/, no oracle pin and not the input generator imports the library
    package (the generator is a module of its own at the repository root)."""
    files = sorted((ROOT / "oracle").glob("*.py")) + [ROOT / "tests" / "test_oracle.py",
                                                        ROOT / "tests" / "relabel.py",
                                                        ROOT / "workloads.py"]
    for path in files:
        assert "paged_kv_cache_459_b200" not in _imports(path), path.name
        assert "paged_kv_cache_459_b200" not in path.read_text(), path.name
    assert "oracle" not in _imports(ROOT / "workloads.py")


def test_library_never_imports_the_oracle():
    """No product file (the package's Python or C/CUDA sources) reaches oracle/."""
    pkg = ROOT / "paged_kv_cache_459_b200"
    for path in sorted(pkg.rglob("*.py")):
        assert "oracle" not in _imports(path), path.name
    for path in SOURCES:
        assert "oracle" not in _code(path).lower(), path.name
