"""Host logic of bench.py that needs no GPU."""


def test_kernel_hash_ignores_comments():
    """The profile key (hash of the device-code sources) changes with code, not comments."""
    import bench
    a = "int f(int x) {  // doubles x\n    return 2 * x; /* twice */\n}\n"
    b = "// header\nint f(int x) {\n\n    return 2 * x;\n}\n"
    c = "int f(int x) {\n    return 3 * x;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
