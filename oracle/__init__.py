"""fp64 CPU oracle for gated retention.  Test infrastructure: used by tests/, the smoke check and
the benchmark's CPU-baseline leg only; the library never imports it."""
