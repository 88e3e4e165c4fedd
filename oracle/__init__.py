"""fp64 CPU oracle of the chunked H2O step. Test infrastructure only: used by
tests/, the smoke check and the benchmark's CPU-baseline leg, never by the
product package."""
