"""fp64 CPU oracle of the MoBA prefill forward pass: test infrastructure, never the product path."""
