"""Float64 CPU oracle (test infrastructure only; never used by the product
path).  See powersgd64.py for the method and philox64.py for the seeded
initial-Q draw."""
